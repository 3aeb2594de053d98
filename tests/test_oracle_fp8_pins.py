"""Pins for the oracle's FP8 (E4M3) functions (CPU only).

The FP8 variant of W8A8 is named by the Red Hat W8A8 article ("When W8A8 INT8 quantization
is a good fit", "What to explore next") and the inference-engineering notes ("05
Quantization AWQ GPTQ FP8", "Ladder"); neither fixes the encoding, so the oracle takes OCP
E4M3 (no infinities, largest finite 448) with round-to-nearest-even and saturation, and
scales absmax / 448. These pins tie that reading to the format's closed form, to torch's own
float8_e4m3fn conversion (a library routine), and to exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_smoothed_b200 import synth


def torch_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).float().numpy()


def torch_encode(v: np.ndarray) -> np.ndarray:
    """torch's RN-even conversion; it does not saturate, so values are clipped to +-448
    first (clipping commutes with rounding to a format whose largest value is 448)."""
    v = np.clip(np.asarray(v, dtype=np.float32), -448.0, 448.0)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def closed_form(c: int) -> float:
    sign = -1.0 if c & 0x80 else 1.0
    e, f = (c >> 3) & 15, c & 7
    if e == 0:
        return sign * f * 2.0 ** -9
    return sign * (1.0 + f / 8.0) * 2.0 ** (e - 7)


def test_decode_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle.e4m3_to_f32(int(c)) for c in codes])
    lib = torch_decode(codes)
    for c in range(256):
        if c & 0x7F == 0x7F:
            assert np.isnan(ours[c]) and np.isnan(lib[c])
        else:
            assert ours[c] == lib[c] == closed_form(c), hex(c)
    assert ours[0x7E] == 448.0 and ours[0x38] == 1.0 and ours[0x08] == 2.0 ** -6
    assert ours[0x01] == 2.0 ** -9 and ours[0xFE] == -448.0


def test_encode_roundtrip_midpoints_and_saturation():
    finite = [c for c in range(128) if c != 0x7F]
    for c in finite:
        v = oracle.e4m3_to_f32(c)
        assert oracle.f32_to_e4m3(v) == c
        assert oracle.f32_to_e4m3(-v) == c | 0x80
    for c in finite[:-1]:
        a, b = oracle.e4m3_to_f32(c), oracle.e4m3_to_f32(c + 1)
        mid = (a + b) / 2.0  # exact in binary32 (five significant bits)
        assert np.float32(mid) == mid
        even = c if c % 2 == 0 else c + 1
        assert oracle.f32_to_e4m3(mid) == even, hex(c)
        below = float(np.nextafter(np.float32(mid), np.float32(0)))
        above = float(np.nextafter(np.float32(mid), np.float32(1e9)))
        assert oracle.f32_to_e4m3(below) == c
        assert oracle.f32_to_e4m3(above) == c + 1
        assert oracle.f32_to_e4m3(-above) == (c + 1) | 0x80
    for v in (448.0, 448.5, 463.99, 464.0, 480.0, 1e30, float("inf")):
        assert oracle.f32_to_e4m3(v) == 0x7E
        assert oracle.f32_to_e4m3(-v) == 0xFE
    assert oracle.f32_to_e4m3(float("nan")) & 0x7F == 0x7F
    assert oracle.f32_to_e4m3(0.0) == 0x00 and oracle.f32_to_e4m3(-0.0) == 0x80
    # below half the smallest subnormal: zero; exactly half: tie to even (zero)
    assert oracle.f32_to_e4m3(2.0 ** -10) == 0x00
    assert oracle.f32_to_e4m3(float(np.nextafter(np.float32(2.0 ** -10), np.float32(1)))) == 0x01
    assert oracle.f32_to_e4m3(3 * 2.0 ** -10) == 0x02


@pytest.mark.parametrize("seed", [0, 1])
def test_encode_matches_torch(seed):
    rng = np.random.default_rng(seed)
    v = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(100.0),
        rng.standard_normal(4000).astype(np.float32) * np.float32(2.0 ** -8),
        rng.uniform(-500, 500, 2000).astype(np.float32),
    ])
    ours = np.array([oracle.f32_to_e4m3(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(ours, torch_encode(v))


def test_quantize_row_recovers_exact_codes():
    """A row y = decode(c) * 2^t with some |c| = 448 has s = 2^t exactly and q = c: pins the
    divisor 448, the use of the row's own absmax and the element order."""
    rng = np.random.default_rng(3)
    for t in (-20, -3, 0, 7):
        codes = rng.integers(0, 256, 300).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x10
        codes[17] = 0xFE
        codes[(codes & 0x7F) == 0x00] = 0x00  # canonical +0 (a -0 input maps to code 0x80)
        y = np.array([oracle.e4m3_to_f32(int(c)) for c in codes], np.float32) * np.float32(2.0 ** t)
        q, s = oracle.quantize_row_f32_fp8(y)
        assert s == np.float32(2.0 ** t)
        assert np.array_equal(q, codes)


@pytest.mark.parametrize("seed", [0, 5])
def test_quantize_row_matches_library_division_and_bounds(seed):
    rng = np.random.default_rng(seed)
    y = (rng.standard_normal(2048) * np.exp(rng.uniform(-8, 3, 2048))).astype(np.float32)
    y[5] = -37.25
    q, s = oracle.quantize_row_f32_fp8(y)
    amax = np.float32(np.max(np.abs(y)))
    assert s == amax / np.float32(448.0)
    assert np.array_equal(q, torch_encode(y / np.float32(s)))
    assert q[np.argmax(np.abs(y))] in (0x7E, 0xFE)
    deq = torch_decode(q).astype(np.float64) * float(s)
    err = np.abs(deq - y.astype(np.float64))
    normal = np.abs(y / s) >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(y[normal]) * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * float(s) * (1 + 1e-6))


def test_zero_row_and_sign_of_zero():
    q, s = oracle.quantize_row_f32_fp8(np.zeros(64, np.float32))
    assert s == 0.0 and not q.any()
    q, s = oracle.quantize_row_f32_fp8(np.array([-1e-30, 1.0, -1.0], np.float32))
    assert list(q) == [0x80, 0x7E, 0xFE]


def test_quantize_rows_fp8_with_sinv_and_weights():
    x = synth.activation(5, 256, 11)
    sinv = np.random.default_rng(2).uniform(0.25, 4.0, 256).astype(np.float32)
    q, s = oracle.quantize_rows_fp8(x, sinv)
    y = oracle.bf16_to_f32(x) * sinv[None, :]
    for m in range(5):
        amax = np.float32(np.max(np.abs(y[m])))
        assert s[m] == amax / np.float32(448.0)
        assert np.array_equal(q[m], torch_encode(y[m] / s[m]))
    q2, s2 = oracle.quantize_rows_f32_fp8(y)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    # weights: rows are output channels of W diag(s); with s = 1 it is the bf16 weight itself
    w = synth.weight(7, 128, 4)
    wq, sch = oracle.rtn_weights_fp8(w)
    wf = oracle.bf16_to_f32(w)
    for n in range(7):
        assert sch[n] == np.float32(np.max(np.abs(wf[n]))) / np.float32(448.0)
        assert np.array_equal(wq[n], torch_encode(wf[n] / sch[n]))


def test_fp8_rmsnorm_and_silu_quantize_their_fp32_rows():
    x = synth.activation(3, 512, 21)
    gamma = np.random.default_rng(8).uniform(0.5, 2.0, 512).astype(np.float32)
    r = oracle.smooth_rmsnorm_quant_fp8(x, gamma, 1e-5)
    ri = oracle.smooth_rmsnorm_quant(x, gamma, 1e-5, want_y=True)
    assert np.array_equal(r["y"], ri["y"])
    for m in range(3):
        assert r["s"][m] == np.float32(np.max(np.abs(ri["y"][m]))) / np.float32(448.0)
        assert np.array_equal(r["q"][m], torch_encode(ri["y"][m] / r["s"][m]))
    gu = synth.activation(3, 2 * 384, 22)
    q, s = oracle.silu_mul_quant_fp8(gu)
    a = oracle.silu_mul(gu)
    for m in range(3):
        assert np.array_equal(q[m], torch_encode(a[m] / s[m]))


def test_gemm_fp8_brute_force():
    rng = np.random.default_rng(9)
    M, N, K = 3, 5, 67

    def codes(shape):
        c = rng.integers(0, 256, shape).astype(np.uint8)
        c[(c & 0x7F) == 0x7F] = 0x3A
        return c

    xq, wq = codes((M, K)), codes((N, K))
    st = rng.uniform(0.01, 2.0, M).astype(np.float32)
    sc = rng.uniform(0.01, 2.0, N).astype(np.float32)
    y, acc, absacc = oracle.gemm_fp8(xq, st, wq, sc)
    xf = [[Fraction(oracle.e4m3_to_f32(int(c))) for c in row] for row in xq]
    wf = [[Fraction(oracle.e4m3_to_f32(int(c))) for c in row] for row in wq]
    for m in range(M):
        for n in range(N):
            exact = sum(a * b for a, b in zip(xf[m], wf[n]))
            assert Fraction(acc[m, n]) == exact  # the binary64 sum is exact
            assert Fraction(absacc[m, n]) == sum(abs(a * b) for a, b in zip(xf[m], wf[n]))
            f = np.float32(np.float32(np.float32(float(exact)) * st[m]) * sc[n])
            ref = torch.tensor([float(f)], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
            assert int(y[m, n]) == int(ref.item()) & 0xFFFF
    # transposed operands give the transposed accumulator
    _, acc_t, _ = oracle.gemm_fp8(wq, sc, xq, st)
    assert np.array_equal(acc_t, acc.T)


def test_dequant_f32acc_matches_the_gemm_epilogue():
    """With exactly representable accumulators the epilogue alone equals the GEMM's."""
    rng = np.random.default_rng(12)
    xq = rng.integers(0x20, 0x40, (4, 32)).astype(np.uint8)  # small codes: sums exact in f32
    wq = rng.integers(0x20, 0x40, (6, 32)).astype(np.uint8)
    st = rng.uniform(0.1, 1.0, 4).astype(np.float32)
    sc = rng.uniform(0.1, 1.0, 6).astype(np.float32)
    y, acc, _ = oracle.gemm_fp8(xq, st, wq, sc)
    assert np.array_equal(acc.astype(np.float32).astype(np.float64), acc)
    assert np.array_equal(oracle.dequant_f32acc(acc.astype(np.float32), st, sc), y)
    a = np.float32(3.0)
    want = torch.tensor([float(np.float32(np.float32(a * st[1]) * sc[2]))]).to(torch.bfloat16)
    got = oracle.dequant_f32acc(np.full((4, 6), a, np.float32), st, sc)[1, 2]
    assert int(got) == int(want.view(torch.int16).item()) & 0xFFFF
