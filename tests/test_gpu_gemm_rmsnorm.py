"""Parity of the o projection's GEMM followed by the residual add and the smoothed RMSNorm with
per-token quantization (w8a8_gemm_rmsnorm_quant) with the oracle's chain: y bit for bit
against the oracle's GEMM + dequant, h = bf16(y + residual) bit for bit, and q, s of every row
exactly (a row whose binary64 mean of squares lies next to a binary32 rounding boundary may
take either neighbour, the method leaving the summation order free). Both forms are covered:
the GEMM followed by the row kernel (the default), and one launch (the cluster split-K GEMM
whose last CTAs run the row pass: M <= 64, N <= 8192)."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import synth
from helpers import assert_rms_rows_match, bf16_out, dev, dev_bf16, host, host_bf16, i8_out

pytestmark = pytest.mark.gpu

EPS = 1e-5


def _inputs(M, N, K, seed):
    xq = synth.int8_codes((M, K), seed)
    wq = synth.int8_codes((N, K), seed + 1)
    # scales that keep y of the order of the residual stream
    st = synth.scales(M, seed + 2, 1e-3, 1e-2)
    sc = synth.scales(N, seed + 3, 1e-4, 1e-3)
    res = synth.activation(M, N, seed + 4)
    gf = synth.gamma(N, seed + 5)
    return xq, st, wq, sc, res, gf


def _run_and_check(M, N, K, seed, ws, inplace=False, one_launch=False):
    xq, st, wq, sc, res, gf = _inputs(M, N, K, seed)
    y_ref, _ = oracle.gemm_dequant(xq, st, wq, sc, want_acc=False)
    r = dev_bf16(res)
    y, y_check = bf16_out((M, N))
    q, q_check = i8_out((M, N))
    q, s, h, y = w8.w8a8_gemm_rmsnorm_quant(dev(xq), dev(st), dev(wq), dev(sc), r, dev(gf), EPS,
                                            y=y, q=q, h_out=r if inplace else None,
                                            workspace=ws, one_launch=one_launch)
    torch.cuda.synchronize()
    assert w8.w8a8_last_device_status(torch.cuda.current_stream()) == 0
    y_check()
    q_check()
    yh = host_bf16(y)
    assert np.array_equal(yh, y_ref)
    ref, _ = assert_rms_rows_match(host(q), host(s), yh, gf, EPS, residual=res)
    assert np.array_equal(host_bf16(h), ref["h"])
    if inplace:
        assert h.data_ptr() == r.data_ptr()


# (M, N, K): token counts across the token tiles of 16 / 32 / 64, rows of up to 4096 and of
# up to 8192 values (N = 4352: 34 channel blocks, a row not a multiple of 1024), K of 512 ..
# 4096 with a ragged last k-block (K = 4112)
ONE_LAUNCH_SHAPES = [(1, 4096, 4096), (2, 4096, 4096), (7, 1024, 2048), (16, 4096, 1024),
                     (17, 2048, 4096), (33, 4096, 512), (64, 4096, 4096), (5, 8192, 1024),
                     (64, 6144, 2048), (3, 4352, 4112)]
# M > 64 (tile kernels), N > 8192, and K = 128 (one k-block: the stream-K plan)
OTHER_SHAPES = [(100, 4096, 1024), (4, 12288, 512), (65, 1024, 1024), (3, 1024, 128)]


@pytest.mark.parametrize("one_launch", [True, False])
@pytest.mark.parametrize("M,N,K", ONE_LAUNCH_SHAPES)
def test_decode_shapes_match_oracle_chain(M, N, K, one_launch):
    assert w8.w8a8_gemm_rmsnorm_quant_one_launch_ok(M, N, K)
    ws = w8.Workspace()
    for call in range(2):  # the second call finds the tail's counters zeroed by the first
        _run_and_check(M, N, K, seed=M + N + K + call, ws=ws, one_launch=one_launch)
    assert int(torch.count_nonzero(ws.buf[:4096])) == 0, "flag words left set"


@pytest.mark.parametrize("M,N,K", OTHER_SHAPES)
def test_other_shapes_match_oracle_chain(M, N, K):
    assert not w8.w8a8_gemm_rmsnorm_quant_one_launch_ok(M, N, K)
    _run_and_check(M, N, K, seed=3 * M + N + K, ws=w8.Workspace())
    xq, st, wq, sc, res, gf = _inputs(M, N, K, 9)
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED_SHAPE"):
        w8.w8a8_gemm_rmsnorm_quant(dev(xq), dev(st), dev(wq), dev(sc), dev_bf16(res), dev(gf),
                                   EPS, one_launch=True)


@pytest.mark.parametrize("one_launch", [True, False])
@pytest.mark.parametrize("M", [1, 16, 64])
def test_in_place_residual(M, one_launch):
    _run_and_check(M, 4096, 2048, seed=M + 5, ws=w8.Workspace(), inplace=True,
                   one_launch=one_launch)


def test_one_launch_equals_separate_gpu_calls():
    """The one launch and the chain of the two separate entry points give the same bits (the
    order-free RMSNorm sum aside, which the two take in different orders: compared here on
    rows the oracle marks unambiguous)."""
    M, N, K = 16, 4096, 4096
    xq, st, wq, sc, res, gf = _inputs(M, N, K, 11)
    args = (dev(xq), dev(st), dev(wq), dev(sc))
    q1, s1, h1, y1 = w8.w8a8_gemm_rmsnorm_quant(*args, dev_bf16(res), dev(gf), EPS,
                                                one_launch=True)
    y0 = w8.w8a8_gemm_dequant(*args)
    q0, s0, h0 = w8.w8a8_smooth_rmsnorm_quant(y0, dev(gf), EPS, residual=dev_bf16(res))
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(h0.view(torch.int16), h1.view(torch.int16))
    amb = oracle.smooth_rmsnorm_quant(host_bf16(y0), gf, EPS, residual=res)["ambiguous"]
    keep = torch.from_numpy(~amb).cuda()
    assert torch.equal(q0[keep], q1[keep]) and torch.equal(s0[keep], s1[keep])


def test_shared_workspace_with_stream_k_gemms():
    """One workspace serves stream-K GEMMs (flag words 0 .. grid - 1) and the one-launch call
    (counter words 1022 and 1023), interleaved, each finding the words it needs zero."""
    ws = w8.Workspace()
    for i, (M, N) in enumerate(((64, 16384), (7, 20480))):
        xq, st, wq, sc, _, _ = _inputs(M, N, 4096, 40 + i)
        y = w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), variant=2, workspace=ws)
        y_ref, _ = oracle.gemm_dequant(xq, st, wq, sc, want_acc=False)
        assert np.array_equal(host_bf16(y), y_ref)
        _run_and_check(9 + i, 4096, 4096, seed=50 + i, ws=ws, one_launch=True)
    assert int(torch.count_nonzero(ws.buf[:4096])) == 0


def test_argument_errors():
    M, N, K = 4, 1024, 512
    xq, st, wq, sc, res, gf = _inputs(M, N, K, 1)
    a = (dev(xq), dev(st), dev(wq), dev(sc))
    r = dev_bf16(res)
    with pytest.raises(w8.W8A8Error, match="INVALID_ARG"):
        w8.w8a8_gemm_rmsnorm_quant(*a, r, dev(gf), -1.0)
    with pytest.raises(w8.W8A8Error, match="INVALID_ARG"):  # y may not alias the residual
        w8.w8a8_gemm_rmsnorm_quant(*a, r, dev(gf), EPS, y=r)
    with pytest.raises(w8.W8A8Error, match="WORKSPACE"):
        w8.w8a8_gemm_rmsnorm_quant(*a, r, dev(gf), EPS,
                                   workspace=torch.zeros(1024, dtype=torch.uint8, device="cuda"))
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED_SHAPE"):  # row length N % 16 != 0
        xq2, st2, wq2, sc2, res2, gf2 = _inputs(M, 1032, K, 2)
        w8.w8a8_gemm_rmsnorm_quant(dev(xq2), dev(st2), dev(wq2), dev(sc2), dev_bf16(res2),
                                   dev(gf2), EPS)
