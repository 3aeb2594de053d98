"""The no-allocation GEMM entry point (w8a8_gemm_dequant_noalloc), for callers that cannot
allocate device memory (a plugin inside another runtime's launch path, a fixed memory
budget, a stream under capture). It must give the oracle's output and the same output as
w8a8_gemm_dequant, call after call, using only its built-in 8 MiB scratch array.

This file is collected last on purpose, and passes both alone in a fresh process and after
the rest of the suite."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
from int8_w8a8_quantized_smoothed_b200 import synth
import oracle

pytestmark = pytest.mark.gpu


def _ulp(a, b):
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(ordered(a) - ordered(b))


def _bits(y):
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _noalloc_scratch_bytes(M, N, K):
    """Scratch bytes the entry point needs: it always takes the small-M kernels, cluster
    split-K for few 128-channel blocks and stream-K for many, as w8a8_gemm_dequant does
    for M <= 64."""
    nb, kb = -(-N // 128), -(-K // 128)
    variant = 3 if (2 * nb <= _sms() and kb >= 2) else 2
    return w8.w8a8_gemm_workspace_size_ex(M, N, K, variant, 0, 0)


# Stream-K shapes whose CTA shares end inside channel blocks: their partial sums go through
# the scratch array (M = 108 is the largest token count whose scratch fits on 148 SMs).
SCRATCH_SHAPES = [(16, 20480, 1024), (100, 10240, 2048), (108, 20480, 1024)]
# Shapes that need no scratch: stream-K with whole channel blocks per CTA (the first), and
# cluster split-K (the rest).
PLAIN_SHAPES = [(64, 28672, 4096), (8, 6144, 4096), (64, 4096, 14336), (1, 512, 256),
                (33, 1032, 4096)]


@pytest.mark.parametrize("M,N,K", SCRATCH_SHAPES + PLAIN_SHAPES)
def test_noalloc_matches_oracle_and_gemm_dequant_twice(M, N, K):
    dev = torch.device("cuda", 0)
    need = _noalloc_scratch_bytes(M, N, K)
    if (M, N, K) in SCRATCH_SHAPES:
        assert 0 < need <= w8.NOALLOC_SCRATCH_BYTES, "shape meant to use the scratch array"
    else:
        assert need == 0
    xq_h = synth.int8_codes((M, K), M + K)
    wq_h = synth.int8_codes((N, K), N + K)
    st_h = synth.scales(M, 1, 1e-3, 0.5)
    sc_h = synth.scales(N, 2, 1e-4, 2e-2)
    y_ref, _ = oracle.gemm_dequant(xq_h, st_h, wq_h, sc_h, want_acc=False)
    xq, wq = torch.from_numpy(xq_h).to(dev), torch.from_numpy(wq_h).to(dev)
    st, sc = torch.from_numpy(st_h).to(dev), torch.from_numpy(sc_h).to(dev)
    lib_ref = _bits(w8.w8a8_gemm_dequant(xq, st, wq, sc))
    assert np.array_equal(lib_ref, y_ref)
    for _ in range(2):  # the scratch keeps the last call's contents between calls
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        w8.w8a8_gemm_dequant_noalloc(xq, st, wq, sc, y=y)
        torch.cuda.synchronize()
        got = _bits(y)
        assert _ulp(got, y_ref).max() <= 1
        assert np.array_equal(got, y_ref)
        assert np.array_equal(got, lib_ref)
    assert w8.w8a8_device_status(reset=True) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    dev = torch.device("cuda", 0)
    N, K = 20480, 1024
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    sc = torch.ones(N, device=dev)
    # one split stream-K slot per SM: 512 bytes per token of the (rounded) token count
    M = 112
    assert _noalloc_scratch_bytes(M, N, K) == 4096 + _sms() * 128 * M * 4
    if _sms() == 148:
        assert _noalloc_scratch_bytes(M, N, K) > w8.NOALLOC_SCRATCH_BYTES
        assert _noalloc_scratch_bytes(108, N, K) <= w8.NOALLOC_SCRATCH_BYTES
    for M in (112, 256):
        if _noalloc_scratch_bytes(M, N, K) <= w8.NOALLOC_SCRATCH_BYTES:
            continue
        xq = torch.zeros((M, K), dtype=torch.int8, device=dev)
        with pytest.raises(w8.W8A8Error, match="WORKSPACE"):
            w8.w8a8_gemm_dequant_noalloc(xq, torch.ones(M, device=dev), wq, sc)
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED"):
        w8.w8a8_gemm_dequant_noalloc(torch.zeros((257, K), dtype=torch.int8, device=dev),
                                     torch.ones(257, device=dev), wq, sc)
