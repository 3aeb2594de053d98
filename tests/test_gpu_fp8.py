"""Parity of the FP8 (E4M3) variant with the oracle, through the C ABI.

Row kernels (quantize_rows, smoothed RMSNorm, SiLU*up): E4M3 codes and fp32 scales
bit-exact. GEMM: the tensor cores add the exact E4M3 products in binary32 in an order of
their own, so the accumulator is checked against the exact sum within the worst-case bound
of any binary32 summation of K terms, |acc - exact| <= gamma * sum|products| with
gamma = (K + 16) * 2^-24 (K additions inside the MMA chain plus the split-K merges), and the
bf16 output is checked bit-exactly against the epilogue applied to the device's own
accumulator. Sums whose every partial sum is representable in binary32 must come out exact.
Beside that guaranteed bound, an empirical guard: the error must stay within
ACC_GUARD_UNITS units of 2^-24 * sum|products| (measured on B200: at most 14 units at K up to
16384), so a systematic accumulation slip far below the worst-case bound still fails.
"""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import prep, synth
from helpers import assert_rms_rows_match, dev, dev_bf16, f32_out, host, host_bf16, with_canary

pytestmark = pytest.mark.gpu
ACC_GUARD_UNITS = 64.0

ROW_SHAPES = [(1, 16), (3, 48), (16, 256), (37, 4096), (5, 8192), (64, 14336), (3, 28672),
              (2, 32768), (300, 4096), (7, 4112)]


def fp8_out(shape):
    t, check = with_canary(shape, torch.uint8, 0x7F)  # 0x7F is a NaN code: never written
    return t.view(w8.FP8), check


def codes(t):
    return t.view(torch.uint8).cpu().numpy()


def dev_fp8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda().view(w8.FP8)


def _sinv(K, seed):
    return (1.0 / np.abs(synth.gamma(K, seed))).astype(np.float32)


@pytest.mark.parametrize("M,K", ROW_SHAPES)
@pytest.mark.parametrize("smooth", [False, True])
def test_quantize_rows_fp8_bit_exact(M, K, smooth):
    x = synth.activation(M, K, seed=M * 5 + K)
    sinv = _sinv(K, K + 1) if smooth else None
    q_ref, s_ref = oracle.quantize_rows_fp8(x, sinv)
    q, cq = fp8_out((M, K))
    s, cs = f32_out((M,))
    w8.w8a8_quantize_rows_fp8(dev_bf16(x), None if sinv is None else dev(sinv), q=q, s_tok=s)
    torch.cuda.synchronize()
    cq(); cs()
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(codes(q), q_ref)


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_quantize_rows_fp8_midpoints_zero_and_tiny_rows():
    """Row 0 has amax 448, so s = 1 and every value is quantized as itself: E4M3 rounding
    midpoints (ties to even) and their bf16 neighbours drive the exact-quotient fallback.
    Row 1 is all zero (s = 0, codes +0); rows 2-3 have scales below 2^-100."""
    K = 1024
    vals = [oracle.e4m3_to_f32(c) for c in range(0x7E)]
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    row0 = [448.0]
    for m in mids:
        b = float(torch.tensor(m).to(torch.bfloat16))
        up = float(np.frombuffer((np.array([b], np.float32).view(np.uint32) + (1 << 16))
                                 .astype(np.uint32).tobytes(), np.float32)[0])
        dn = float(np.frombuffer((np.array([b], np.float32).view(np.uint32) - (1 << 16))
                                 .astype(np.uint32).tobytes(), np.float32)[0])
        row0 += [m, -m, up, dn]
    row0 = (row0 + [0.0] * K)[:K]
    rng = np.random.default_rng(3)
    rows = [row0, [0.0] * K, list(rng.standard_normal(K) * 1e-36),
            list(rng.standard_normal(K) * 1e-32)]
    x = np.stack([_bf16(r) for r in rows])
    q_ref, s_ref = oracle.quantize_rows_fp8(x)
    assert s_ref[0] == 1.0 and s_ref[1] == 0.0 and (s_ref[2:] < 2.0 ** -100).all()
    q, s = w8.w8a8_quantize_rows_fp8(dev_bf16(x))
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(codes(q), q_ref)


@pytest.mark.parametrize("M,K", [(1, 16), (16, 4096), (37, 4096), (5, 8192), (300, 4112),
                                 (2, 32768)])
@pytest.mark.parametrize("res", [False, True])
def test_smooth_rmsnorm_quant_fp8(M, K, res):
    x = synth.activation(M, K, seed=K + M + 11)
    gamma = (synth.gamma(K, K) * _sinv(K, 3)).astype(np.float32)
    r = synth.activation(M, K, seed=K + 3) if res else None
    out = w8.w8a8_smooth_rmsnorm_quant_fp8(dev_bf16(x), dev(gamma), 1e-5,
                                           residual=None if r is None else dev_bf16(r))
    q, s = out[0], out[1]
    ref, _ = assert_rms_rows_match(codes(q), host(s), x, gamma, 1e-5, residual=r,
                                   ref_fn=oracle.smooth_rmsnorm_quant_fp8)
    if res:
        assert np.array_equal(host_bf16(out[2]), ref["h"])


@pytest.mark.parametrize("M,I", [(1, 16), (16, 14336), (37, 4096), (300, 1024), (3, 28672)])
def test_silu_mul_quant_fp8(M, I):
    gu = synth.normal_bf16((M, 2 * I), seed=M + I + 1, std=2.5)
    q_ref, s_ref = oracle.silu_mul_quant_fp8(gu)
    q, cq = fp8_out((M, I))
    s, cs = f32_out((M,))
    w8.w8a8_silu_mul_quant_fp8(dev_bf16(gu), q=q, s_tok=s)
    torch.cuda.synchronize()
    cq(); cs()
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(codes(q), q_ref)


def test_weight_prep_fp8_through_quantize_rows():
    N, K = 96, 4096
    w = synth.weight(N, K, 19)
    s_fac = (1.0 / _sinv(K, 20)).astype(np.float32)
    wq_ref, sch_ref = oracle.rtn_weights_fp8(w, s_fac)
    wq, sch = w8.w8a8_quantize_rows_fp8(dev_bf16(w), dev(s_fac))
    assert np.array_equal(codes(wq), wq_ref) and np.array_equal(host(sch), sch_ref)


# ---------------------------------------------------------------------------- GEMM
#
# variant 1 = persistent tile kernel (tile_n 128 / 256 / 512 = CTA pair), 2 = swap-AB
# stream-K (binary32 partials through the workspace), 3 = swap-AB cluster split-K (binary32
# partials read from the cluster's shared memory and added in rank order)

def _operands(M, N, K, seed):
    x = synth.activation(M, K, seed)
    w = synth.weight(N, K, seed + 1)
    xq, s_tok = oracle.quantize_rows_fp8(x)
    wq, s_ch = oracle.rtn_weights_fp8(w)
    return xq, s_tok, wq, s_ch


def _check_gemm(xq, s_tok, wq, s_ch, variant=0, ctas=0, tile_n=0, exact=False):
    M, K = xq.shape
    N = wq.shape[0]
    y_ref, acc_ref, absacc = oracle.gemm_fp8(xq, s_tok, wq, s_ch)
    acc, cacc = with_canary((M, N), torch.float32, float("nan"))
    y = w8.w8a8_gemm_dequant_fp8(dev_fp8(xq), dev(s_tok), dev_fp8(wq), dev(s_ch), acc_out=acc,
                                 variant=variant, ctas=ctas, tile_n=tile_n)
    torch.cuda.synchronize()
    cacc()
    a = host(acc).astype(np.float64)
    err = np.abs(a - acc_ref)
    if exact:
        assert np.array_equal(a, acc_ref), f"max err {err.max()}"
    gamma = (K + 16) * 2.0 ** -24
    bound = gamma * absacc
    worst = float((err / np.maximum(absacc, 1e-300)).max())
    assert (err <= bound).all(), f"acc error {worst:.3g} x sum|p| exceeds {gamma:.3g}"
    assert worst <= ACC_GUARD_UNITS * 2.0 ** -24, f"acc error {worst * 2 ** 24:.1f} units"
    assert np.array_equal(host_bf16(y), oracle.dequant_f32acc(host(acc), s_tok, s_ch))
    # and the output is the exact result's wherever the accumulator rounding did not matter
    same = err == 0
    assert np.array_equal(host_bf16(y)[same], y_ref[same])
    return worst


GEMM_CASES = [
    # (M, N, K, variant, ctas, tile_n); tile_n 512 with ctas > 0: stream-K over that many
    # CTA pairs (binary32 partials of split tiles added by the owner pair)
    (300, 1000, 512, 1, 24, 512),
    (512, 4096, 4096, 1, 74, 512),
    (257, 264, 4112, 1, 5, 512),
    (1, 4096, 4096, 0, 0, 0),
    (16, 6144, 4096, 0, 0, 0),
    (37, 1024, 4112, 2, 0, 0),
    (64, 2048, 1024, 2, 37, 0),
    (64, 520, 4096, 2, 0, 0),
    (200, 512, 2048, 2, 0, 0),
    (520, 256, 1024, 2, 0, 0),
    (300, 1000, 512, 1, 0, 128),
    (300, 1000, 512, 1, 0, 256),
    (300, 1000, 512, 1, 0, 512),
    (512, 1024, 1024, 0, 0, 0),
    (129, 264, 16, 1, 0, 0),
    (16, 4096, 4096, 3, 0, 0),
    (64, 6144, 4096, 3, 3, 0),
    (37, 1024, 4112, 3, 8, 0),
    (300, 512, 1024, 3, 0, 0),
    (1, 256, 14336, 3, 5, 0),
]


@pytest.mark.parametrize("M,N,K,variant,ctas,tile_n", GEMM_CASES)
def test_gemm_fp8(M, N, K, variant, ctas, tile_n):
    ops = _operands(M, N, K, seed=M + N + K)
    _check_gemm(*ops, variant=variant, ctas=ctas, tile_n=tile_n)


@pytest.mark.parametrize("variant,tile_n", [(1, 128), (1, 512), (2, 0), (3, 0)])
def test_gemm_fp8_exact_when_partial_sums_fit(variant, tile_n):
    """Codes with values in [1, 4): products are multiples of 2^-6 below 16, so every partial
    sum of K = 4096 of them is a multiple of 2^-6 below 2^16 and exact in binary32."""
    rng = np.random.default_rng(7)
    M, N, K = 96, 384, 4096

    def small_codes(shape):
        e = rng.integers(7, 9, shape)
        f = rng.integers(0, 8, shape)
        sgn = rng.integers(0, 2, shape) << 7
        return (sgn | (e << 3) | f).astype(np.uint8)

    xq, wq = small_codes((M, K)), small_codes((N, K))
    s_tok = rng.uniform(0.01, 1.0, M).astype(np.float32)
    s_ch = rng.uniform(0.01, 1.0, N).astype(np.float32)
    _check_gemm(xq, s_tok, wq, s_ch, variant=variant, tile_n=tile_n, exact=True)


def test_fp8_linear_chain_matches_oracle():
    """RMSNorm -> FP8 quant -> FP8 GEMM, the decode-shaped linear layer of the FP8 variant."""
    M, K, N = 16, 4096, 6144
    x = synth.activation(M, K, 41)
    gamma = synth.gamma(K, 42)
    w = synth.weight(N, K, 43)
    wq, s_ch = oracle.rtn_weights_fp8(w)
    q, s = w8.w8a8_smooth_rmsnorm_quant_fp8(dev_bf16(x), dev(gamma), 1e-5)
    ref, _ = assert_rms_rows_match(codes(q), host(s), x, gamma, 1e-5,
                                   ref_fn=oracle.smooth_rmsnorm_quant_fp8)
    _check_gemm(codes(q), host(s), wq, s_ch)


# ---------------------------------------------------------------- fused gate|up + SiLU*up
#
# The fused call's binary32 accumulators equal the plain FP8 GEMM's on the same interleaved
# weight under the same plan (the automatic one; the fused call takes stream-K where that
# plan is the cluster split-K, so the reference is asked for stream-K there): SiLU*up and
# the E4M3 quantization of the plain GEMM's bf16 output, by the oracle, must then match the
# fused result bit for bit.

def _gate_up_fp8(M, I, K, seed):
    xq, s_tok = oracle.quantize_rows_fp8(synth.activation(M, K, seed))
    wq, s_ch = oracle.rtn_weights_fp8(synth.weight(2 * I, K, seed + 1))
    return xq, s_tok, wq, s_ch


FUSED_SHAPES = [(1, 1024, 512), (16, 5120, 1024), (64, 14336, 4096), (33, 2048, 1024),
                (8, 128, 4112), (300, 1024, 512), (129, 512, 400), (512, 2048, 1024)]


@pytest.mark.parametrize("M,I,K", FUSED_SHAPES)
def test_fused_gate_up_silu_quant_fp8(M, I, K):
    xq, st, wq, sc = _gate_up_fp8(M, I, K, seed=M + I + K)
    wq_il, sc_il = prep.interleave_gate_up(dev_fp8(wq), dev(sc))
    NB = (2 * I + 127) // 128
    cluster = M <= 64 and 2 * NB <= torch.cuda.get_device_properties(0).multi_processor_count \
        and K > 128
    y_il = w8.w8a8_gemm_dequant_fp8(dev_fp8(xq), dev(st), wq_il, sc_il,
                                    variant=2 if cluster else 0)
    y = host_bf16(y_il).reshape(M, I // 64, 2, 64)
    gu = np.concatenate([y[:, :, 0, :].reshape(M, I), y[:, :, 1, :].reshape(M, I)], axis=1)
    a_ref = oracle.silu_mul(gu)
    q_ref, s_ref = oracle.quantize_rows_f32_fp8(a_ref)
    ws = w8.Workspace()
    for _ in range(2):  # the second call checks that the workspace came back zeroed
        q, s, a = w8.w8a8_gemm_silu_quant_fp8(dev_fp8(xq), dev(st), wq_il, sc_il, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(host(a).view(np.uint32), a_ref.view(np.uint32))
        assert np.array_equal(host(s), s_ref)
        assert np.array_equal(codes(q), q_ref)


def test_fused_fp8_equals_unfused_gpu_chain():
    """Whole channel blocks per CTA (the decode plan for this weight): every accumulator is
    one CTA's sum over all of K in the same order, interleaved or not."""
    M, I, K = 16, 14336, 4096
    xq, st, wq, sc = _gate_up_fp8(M, I, K, 7)
    y = w8.w8a8_gemm_dequant_fp8(dev_fp8(xq), dev(st), dev_fp8(wq), dev(sc))
    q0, s0 = w8.w8a8_silu_mul_quant_fp8(y)
    wq_il, sc_il = prep.interleave_gate_up(dev_fp8(wq), dev(sc))
    q1, s1, _ = w8.w8a8_gemm_silu_quant_fp8(dev_fp8(xq), dev(st), wq_il, sc_il)
    assert torch.equal(q0.view(torch.uint8), q1.view(torch.uint8)) and torch.equal(s0, s1)
