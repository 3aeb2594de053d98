"""Parity of the fused gate|up GEMM + SiLU(gate)*up + per-token quantization
(w8a8_gemm_silu_quant) with the oracle's unfused chain: the gate|up GEMM with dequant to bf16,
then SiLU*up and per-token quantization. a (binary32), the int8 codes and the scales are
compared bit for bit, on decode shapes (cluster split-K and stream-K kernels) and prefill
shapes (one-CTA and CTA-pair tile kernels)."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import prep, synth
from helpers import dev, host

pytestmark = pytest.mark.gpu


def _inputs(M, I, K, seed):
    xq = synth.int8_codes((M, K), seed)
    wq = synth.int8_codes((2 * I, K), seed + 1)
    st = synth.scales(M, seed + 2, 1e-3, 0.5)
    sc = synth.scales(2 * I, seed + 3, 1e-4, 2e-2)
    return xq, st, wq, sc


def _reference(xq, st, wq, sc):
    y = oracle.gemm_dequant(xq, st, wq, sc)[0]
    a = oracle.silu_mul(y)
    q, s = oracle.silu_mul_quant(y)
    return a, q, s


SHAPES = [(1, 1024, 512), (8, 1024, 4096), (33, 2048, 1024), (64, 2048, 4096), (3, 128, 4112),
          (8, 5120, 1024), (64, 5120, 512), (100, 5120, 256),
          (300, 1024, 1024), (129, 512, 400), (1000, 4096, 256)]


@pytest.mark.parametrize("M,I,K", SHAPES)
def test_fused_gate_up_silu_quant_bit_exact(M, I, K):
    xq, st, wq, sc = _inputs(M, I, K, seed=M + I + K)
    a_ref, q_ref, s_ref = _reference(xq, st, wq, sc)
    wq_il, sc_il = prep.interleave_gate_up(dev(wq), dev(sc))
    ws = w8.Workspace()
    for _ in range(2):  # the second call checks that the workspace came back zeroed
        q, s, a = w8.w8a8_gemm_silu_quant(dev(xq), dev(st), wq_il, sc_il, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(host(a).view(np.uint32), a_ref.view(np.uint32))
        assert np.array_equal(host(s), s_ref)
        assert np.array_equal(host(q), q_ref)


def test_fused_equals_unfused_gpu_chain():
    M, I, K = 16, 14336, 4096
    xq, st, wq, sc = _inputs(M, I, K, 7)
    y = w8.w8a8_gemm_dequant(dev(xq), dev(st), dev(wq), dev(sc))
    q0, s0 = w8.w8a8_silu_mul_quant(y)
    wq_il, sc_il = prep.interleave_gate_up(dev(wq), dev(sc))
    q1, s1, _ = w8.w8a8_gemm_silu_quant(dev(xq), dev(st), wq_il, sc_il)
    assert torch.equal(q0, q1) and torch.equal(s0, s1)


def test_shared_workspace_after_other_stream_k_calls():
    """One workspace serves the fused call after stream-K GEMMs of other shapes, whose
    partial-sum slots stay as they were left."""
    ws = w8.Workspace()
    for M, N in ((64, 16384), (7, 4096)):  # dirty the partial slots with two other shapes
        xq, st, wq, sc = _inputs(M, N // 2, 4096, M)
        w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), variant=2, workspace=ws)
    M, I, K = 16, 5120, 4096
    xq, st, wq, sc = _inputs(M, I, K, 3)
    a_ref, q_ref, s_ref = _reference(xq, st, wq, sc)
    wq_il, sc_il = prep.interleave_gate_up(dev(wq), dev(sc))
    q, s, a = w8.w8a8_gemm_silu_quant(dev(xq), dev(st), wq_il, sc_il, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)


def test_stream_k_after_fused_calls_on_the_same_workspace():
    """Small-M fused calls keep each token's group maxima in the workspace past its flag
    words: split stream-K GEMMs issued after them on the same workspace still find their
    flags zero and give the oracle's result."""
    ws = w8.Workspace()
    ws.get(8 << 20)  # one buffer for every call below
    for M, I, K in ((1, 14336, 4096), (16, 5120, 1024)):  # without and with split-K parts
        xq, st, wq, sc = _inputs(M, I, K, 5 + M)
        wq_il, sc_il = prep.interleave_gate_up(dev(wq), dev(sc))
        w8.w8a8_gemm_silu_quant(dev(xq), dev(st), wq_il, sc_il, workspace=ws)
        M2, N2, K2 = 16, 20480, 1024
        assert w8.w8a8_gemm_workspace_size(M2, N2, K2) > 0  # a split stream-K plan
        xq2, st2, wq2, sc2 = _inputs(M2, N2 // 2, K2, 9 + M)
        y = w8.w8a8_gemm_dequant(dev(xq2), dev(st2), dev(wq2), dev(sc2), workspace=ws)
        torch.cuda.synchronize()
        y_ref, _ = oracle.gemm_dequant(xq2, st2, wq2, sc2, want_acc=False)
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), y_ref)
    assert w8.w8a8_device_status(reset=True) == 0


@pytest.mark.parametrize("M,I,K", [(512, 2048, 8192), (300, 512, 16384), (257, 640, 8208)])
def test_fused_silu_on_pair_stream_k(M, I, K):
    """The SiLU*up epilogue on split tiles (these shapes plan stream-K over CTA pairs: few
    tiles, K >= 8192): the owner pair adds the later pieces before it forms a."""
    assert w8.w8a8_gemm_workspace_size(M, 2 * I, K) > 0
    xq, st, wq, sc = _inputs(M, I, K, seed=M + I)
    a_ref, q_ref, s_ref = _reference(xq, st, wq, sc)
    wq_il, sc_il = prep.interleave_gate_up(dev(wq), dev(sc))
    for _ in range(2):
        q, s, a = w8.w8a8_gemm_silu_quant(dev(xq), dev(st), wq_il, sc_il)
        torch.cuda.synchronize()
        assert np.array_equal(host(a).view(np.uint32), a_ref.view(np.uint32))
        assert np.array_equal(host(q), q_ref) and np.array_equal(host(s), s_ref)


def test_interleave_is_a_row_permutation():
    I, K = 192, 32
    wq = torch.arange(2 * I, dtype=torch.int32).repeat_interleave(K).view(2 * I, K)
    w, s = prep.interleave_gate_up(wq, torch.arange(2 * I, dtype=torch.float32))
    order = [*range(0, 64), *range(I, I + 64), *range(64, 128), *range(I + 64, I + 128),
             *range(128, 192), *range(I + 128, I + 192)]
    assert w[:, 0].tolist() == order and s.tolist() == [float(v) for v in order]
