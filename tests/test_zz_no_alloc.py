"""The no-allocation GEMM entry point (w8a8_gemm_dequant_noalloc), for callers that cannot
allocate device memory (a plugin inside another runtime's launch path, a fixed memory
budget, a stream under capture). It must give the same output as w8a8_gemm_dequant, call
after call, using only its built-in 8 MiB scratch array.

This file is collected last on purpose, and passes both alone in a fresh process and after
the rest of the suite."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
from int8_w8a8_quantized_smoothed_b200 import synth

pytestmark = pytest.mark.gpu


def _ulp(a, b):
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(ordered(a) - ordered(b))


def _bits(y):
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


# weights with many 128-channel blocks run the stream-K kernel, whose partial sums go through
# the scratch array; the others run the cluster split-K kernel and need no scratch
SHAPES = [(64, 28672, 4096), (16, 20480, 1024), (100, 10240, 2048), (8, 6144, 4096),
          (64, 4096, 14336), (1, 512, 256), (33, 1032, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_noalloc_matches_gemm_dequant_twice(M, N, K):
    dev = torch.device("cuda", 0)
    xq = torch.from_numpy(synth.int8_codes((M, K), M + K)).to(dev)
    wq = torch.from_numpy(synth.int8_codes((N, K), N + K)).to(dev)
    st = torch.from_numpy(synth.scales(M, 1, 1e-3, 0.5)).to(dev)
    sc = torch.from_numpy(synth.scales(N, 2, 1e-4, 2e-2)).to(dev)
    ref = _bits(w8.w8a8_gemm_dequant(xq, st, wq, sc))
    for _ in range(2):  # the scratch keeps the last call's contents; each call clears it
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        w8.w8a8_gemm_dequant_noalloc(xq, st, wq, sc, y=y)
        torch.cuda.synchronize()
        got = _bits(y)
        assert _ulp(got, ref).max() <= 1
        assert np.array_equal(got, ref)
    assert w8.w8a8_device_status(reset=True) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    dev = torch.device("cuda", 0)
    M, N, K = 256, 20480, 1024  # stream-K scratch 148 CTAs x 256 x 512 B = 19 MB > 8 MiB
    assert w8.w8a8_gemm_workspace_size_ex(M, N, K, 2, 0, 0) > w8.NOALLOC_SCRATCH_BYTES
    xq = torch.zeros((M, K), dtype=torch.int8, device=dev)
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    st = torch.ones(M, device=dev)
    sc = torch.ones(N, device=dev)
    with pytest.raises(w8.W8A8Error, match="WORKSPACE"):
        w8.w8a8_gemm_dequant_noalloc(xq, st, wq, sc)
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED"):
        w8.w8a8_gemm_dequant_noalloc(torch.zeros((257, K), dtype=torch.int8, device=dev),
                                     torch.ones(257, device=dev), wq, sc)
