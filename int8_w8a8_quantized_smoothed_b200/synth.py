"""Seeded synthetic inputs for the W8A8 linear path.

The pages measure on trained Llama-3.1 weights and WikiText-2 / GuideLLM prompts; neither
is available, so seeded random tensors with the same shapes stand in for them:

* activations X [M, K]: N(0, 1), with ceil(1% of K) outlier channels (chosen by a seeded
  permutation) multiplied by 50, rounded to bf16;
* weights W [N, K]: N(0, 0.02^2), rounded to bf16;
* RMSNorm gamma [K]: 1 + N(0, 0.1^2), rounded to bf16 and widened to fp32;
* attention-output stand-in: N(0, 1), rounded to bf16;
* raw int8 codes and positive fp32 scales, for checks of the GEMM on its own.

This module holds none of the method's arithmetic: it only draws numbers. Rounding to
bf16 uses torch's own conversion (round to nearest even). Every generator takes a seed and
returns numpy arrays (bf16 as uint16 bit patterns); the ``*_device`` variants draw on a CUDA
generator for the large benchmark tensors and return torch tensors on that device.
"""
import math

import numpy as np
import torch

OUTLIER_SCALE = 50.0


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def n_outliers(K: int) -> int:
    """Number of outlier channels for a K-channel activation: ceil(1% of K)."""
    return max(1, math.ceil(0.01 * K))


def outlier_channels(K: int, seed: int, count=None) -> np.ndarray:
    count = n_outliers(K) if count is None else count
    perm = torch.randperm(K, generator=_gen(seed + 7919))
    return np.sort(perm[:count].numpy())


def activation(M: int, K: int, seed: int, outliers=None) -> np.ndarray:
    """bf16 [M, K]: N(0,1) with `outliers` channels (default ceil(1% K)) scaled by 50."""
    x = torch.randn(M, K, generator=_gen(seed), dtype=torch.float32)
    if outliers != 0:
        ch = torch.from_numpy(outlier_channels(K, seed, outliers))
        x[:, ch] *= OUTLIER_SCALE
    return _bf16_bits(x)


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * std
    return _bf16_bits(x)


def weight(N: int, K: int, seed: int) -> np.ndarray:
    """bf16 [N, K] ~ N(0, 0.02^2)."""
    return normal_bf16((N, K), seed, 0.02)


def gamma(K: int, seed: int) -> np.ndarray:
    """fp32 [K] = bf16(1 + N(0, 0.1^2))."""
    g = 1.0 + 0.1 * torch.randn(K, generator=_gen(seed), dtype=torch.float32)
    return g.to(torch.bfloat16).to(torch.float32).numpy()


def int8_codes(shape, seed: int, extremes: bool = True) -> np.ndarray:
    """Uniform int8 in [-127, 127]; with `extremes`, row 0 is all +127 and the last row
    alternates -127/+127 so the largest accumulator magnitudes are exercised."""
    q = torch.randint(-127, 128, shape, generator=_gen(seed), dtype=torch.int16)
    q = q.to(torch.int8).numpy()
    if extremes and q.ndim == 2 and q.shape[0] >= 2:
        q[0, :] = 127
        q[-1, :] = np.where(np.arange(q.shape[1]) % 2 == 0, -127, 127)
    return q


def scales(n: int, seed: int, lo: float = 1e-3, hi: float = 1.0) -> np.ndarray:
    """Positive fp32 scales, log-uniform in [lo, hi]."""
    u = torch.rand(n, generator=_gen(seed), dtype=torch.float64)
    v = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    return v.to(torch.float32).numpy()


def row_sample(M: int, seed: int, count: int = 256) -> np.ndarray:
    """A seeded sample of row indices that always includes the first and last row."""
    if M <= count + 2:
        return np.arange(M)
    perm = torch.randperm(M - 2, generator=_gen(seed + 104729))[:count].numpy() + 1
    return np.unique(np.concatenate([[0, M - 1], perm]))


# ------------------------------------------------------------------ device generators


def _dgen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activation_device(M, K, seed, device, outliers=None) -> torch.Tensor:
    x = torch.randn(M, K, generator=_dgen(seed, device), device=device, dtype=torch.float32)
    if outliers != 0:
        ch = torch.from_numpy(outlier_channels(K, seed, outliers)).to(device)
        x[:, ch] *= OUTLIER_SCALE
    return x.to(torch.bfloat16)


def normal_bf16_device(shape, seed, device, std=1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=_dgen(seed, device), device=device,
                    dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def weight_device(N, K, seed, device) -> torch.Tensor:
    return normal_bf16_device((N, K), seed, device, 0.02)


def gamma_device(K, seed, device) -> torch.Tensor:
    g = 1.0 + 0.1 * torch.randn(K, generator=_dgen(seed, device), device=device,
                                dtype=torch.float32)
    return g.to(torch.bfloat16).to(torch.float32)
