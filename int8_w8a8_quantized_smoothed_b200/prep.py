"""Offline preparation of a W8A8 linear (not on the hot path).

SmoothQuant and the weight quantization run once, before serving [W8A8 page, "How we
compressed the model" and "How the SmoothQuant smoothing factor is computed"]:

1. calibration statistics: a_j = max |A[:, j]| over calibration activations entering the
   linear, w_j = max |W[:, j]| over the weight's output channels (column j of W [N, K] is
   input channel j);
2. smoothing factors s_j = a_j^alpha / w_j^(1 - alpha) (binary64, rounded once to binary32;
   s_j = 1 where either maximum is 0);
3. folding: gamma'_j = gamma_j / s_j into a preceding RMSNorm, or 1/s_j applied to X by
   ``w8a8_quantize_rows`` when no norm precedes; the weight's input channel j is scaled by s_j;
4. per-output-channel round-to-nearest int8 weights of the smoothed weight, computed on the
   GPU by ``w8a8_quantize_rows(W, s)`` (each output channel is a row of W).

The calibration statistics and the RMSNorm used to produce calibration activations are plain
torch reductions: they decide only which smoothing factors the benchmark uses, and are
outside the timed path.
"""
import numpy as np
import torch

from . import w8a8_quantize_rows


def column_absmax(t: torch.Tensor) -> torch.Tensor:
    """max over rows of |t[:, j]| as fp32 (exact: a maximum has no rounding)."""
    return t.float().abs().amax(dim=0)


def rmsnorm_calibration(x: torch.Tensor, gamma: torch.Tensor, eps: float) -> torch.Tensor:
    """RMSNorm output x / rms(x) * gamma in fp32: the activation a smoothed linear sees."""
    xf = x.float()
    rstd = torch.rsqrt(xf.pow(2).mean(dim=1, keepdim=True) + eps)
    return xf * rstd * gamma.float()


def smoothing_factors(a_max, w_max, alpha: float) -> np.ndarray:
    a = np.asarray(a_max.detach().cpu() if isinstance(a_max, torch.Tensor) else a_max,
                   dtype=np.float64)
    w = np.asarray(w_max.detach().cpu() if isinstance(w_max, torch.Tensor) else w_max,
                   dtype=np.float64)
    out = np.ones(a.shape, dtype=np.float64)
    ok = (a > 0) & (w > 0)
    out[ok] = np.power(a[ok], alpha) / np.power(w[ok], 1.0 - alpha)
    return out.astype(np.float32)


def fold(gamma, s):
    """gamma' = gamma / s and s_inv = 1 / s, both binary32."""
    s = np.asarray(s, dtype=np.float32)
    g = np.asarray(gamma, dtype=np.float32)
    return (g / s).astype(np.float32), (np.float32(1.0) / s).astype(np.float32)


def quantize_weight(w: torch.Tensor, s: torch.Tensor):
    """int8 [N, K] weights and fp32 [N] per-channel scales of W diag(s), on the GPU."""
    return w8a8_quantize_rows(w, s)


def prepare_linear(w: torch.Tensor, a_max, alpha: float):
    """Smoothing factors from calibration maxima a_max and the weight; returns dict with s
    (numpy), s_inv (numpy) and the device tensors wq, s_ch, s_dev, s_inv_dev."""
    s = smoothing_factors(a_max, column_absmax(w), alpha)
    _, s_inv = fold(np.ones_like(s), s)
    s_dev = torch.from_numpy(s).to(w.device)
    wq, s_ch = quantize_weight(w, s_dev)
    return dict(s=s, s_inv=s_inv, wq=wq, s_ch=s_ch, s_dev=s_dev,
                s_inv_dev=torch.from_numpy(s_inv).to(w.device))


def static_activation_scale(x_cal: torch.Tensor, smooth_inv=None) -> float:
    """Static per-tensor activation scale from a calibration batch [PTQ page, "1. Min-Max
    Calibration"]: S = max(|min|, |max|) / 127 over the (smoothed) calibration values, in
    binary32, for ``w8a8_quantize_rows_static``. The maximum is exact; the division is one
    IEEE binary32 operation."""
    y = x_cal.float()
    if smooth_inv is not None:
        y = y * smooth_inv.float()
    a = y.abs().amax().reshape(1)
    return float((a / torch.tensor([127.0], dtype=torch.float32, device=a.device)).item())


def interleave_gate_up(wq: torch.Tensor, s_ch: torch.Tensor):
    """Row order of the gate|up weight [2I, K] (gate rows 0..I-1, up rows I..2I-1) for
    ``w8a8_gemm_silu_quant``: blocks of 64 gate rows followed by the 64 up rows of the same
    channels, so that each 128-row group holds both halves of 64 output channels. A pure
    permutation of rows (and of their scales)."""
    N, K = wq.shape
    I = N // 2
    if N % 2 or I % 64:
        raise ValueError("the gate|up weight needs 2I rows with I % 64 == 0")
    w = wq.view(2, I // 64, 64, K).permute(1, 0, 2, 3).reshape(N, K).contiguous()
    s = s_ch.view(2, I // 64, 64).permute(1, 0, 2).reshape(N).contiguous()
    return w, s
