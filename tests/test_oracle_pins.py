"""Pins for the oracle (CPU only): the pages' worked examples, closed forms, invariants and
brute force, chosen so that a dropped term, a wrong sign or index, a transposed operand or
the wrong rounding rule in the oracle fails at least one of them."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_smoothed_b200 import synth

F32_EPS = 2.0 ** -23


def f32(x):
    return float(np.float32(x))


def ulp32(x):
    x = abs(np.float32(x))
    return float(np.spacing(x)) if x != 0 else 2.0 ** -149


def round_fraction_to_f32(fr: Fraction) -> float:
    """Exact round-to-nearest-even of a positive rational to binary32 (normal range)."""
    assert fr > 0
    e = math.floor(math.log2(fr.numerator) - math.log2(fr.denominator))
    # fix e so that 2^e <= fr < 2^(e+1)
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    scaled = fr / (Fraction(2) ** (e - 23))  # in [2^23, 2^24)
    lo = math.floor(scaled)
    rem = scaled - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(Fraction(lo) * Fraction(2) ** (e - 23))


# ----------------------------------------------------------------- pages' worked examples


def test_rtn_weight_worked_example(golden):
    g = golden("p2_rtn_weight_example.txt")
    q0, s0 = oracle.quantize_row_f32(g["ch0"])
    q1, s1 = oracle.quantize_row_f32(g["ch1"])
    assert list(q0) == g["codes_ch0_printed"]
    assert list(q1) == g["codes_ch1_formula"]
    # the printed code differs only where the page contradicts its own formula
    assert [a == b for a, b in zip(q1, g["codes_ch1_printed"])] == [True, False, True]
    assert abs(s0 - g["scale_ch0_printed"][0]) < 5e-7
    assert abs(s1 - g["scale_ch1_printed"][0]) < 5e-7
    assert s0 == f32(np.float32(0.74) / np.float32(127.0))


def test_rtn_reconstruction_worked_example(golden):
    g = golden("p2_rtn_weight_example.txt")
    q0, s0 = oracle.quantize_row_f32(g["ch0"])
    rec0 = [int(q) * float(s0) for q in q0]
    for r, p in zip(rec0, g["reconstructed_ch0_printed"]):
        assert abs(r - p) < 5e-5
    x = g["input"]
    out_orig = [sum(a * b for a, b in zip(x, g[c])) for c in ("ch0", "ch1")]
    for o, p in zip(out_orig, g["output_original_printed"]):
        assert abs(o - p) < 5e-4
    out_rec0 = sum(a * b for a, b in zip(x, rec0))
    assert abs(out_rec0 - g["output_reconstructed_ch0_printed"][0]) < 5e-4
    # ch1 with the printed (inconsistent) code reproduces the page's 0.4540: the page's own
    # reconstruction follows from its code, the code does not follow from its formula.
    _, s1 = oracle.quantize_row_f32(g["ch1"])
    assert abs(g["codes_ch1_printed"][1] * float(s1) - g["reconstructed_ch1_printed"][1]) < 5e-5


def test_outlier_activation_worked_example(golden):
    g = golden("p2_outlier_activation.txt")
    q, s = oracle.quantize_row_f32(g["activation"])
    assert list(q) == g["codes_printed"]
    assert abs(s - g["scale_printed"][0]) < 5e-4


def test_smoothed_activation_and_gamma_fold_worked_example(golden):
    g = golden("p2_smoothed_activation.txt")
    norm = np.array(g["normalized"], dtype=np.float32)
    gamma = np.array(g["gamma"], dtype=np.float32)
    act = norm * gamma
    assert np.allclose(act, g["activation_printed"], rtol=0, atol=1e-5)
    q, _ = oracle.quantize_row_f32(act)
    assert list(q) == [1, 1, 1, 127]
    gf, sinv = oracle.fold_gamma(gamma, np.array(g["smoothing"], dtype=np.float32))
    assert list(gf) == g["gamma_smoothed_printed"]
    assert np.allclose(sinv, [1, 1, 1, 0.01], rtol=1e-7)
    act_s = norm * gf
    assert np.allclose(act_s, g["activation_smoothed_printed"], rtol=0, atol=1e-6)
    q, s = oracle.quantize_row_f32(act_s)
    assert list(q) == g["codes_formula"]
    assert abs(s - g["scale_printed"][0]) < 1e-4
    # the page's 63 follows from its rounded scale 0.012 and half-up rounding
    assert math.floor(0.75 / g["scale_printed"][0] + 0.5) == g["codes_printed"][1]


def test_minmax_symmetric_scale(golden):
    g = golden("p3_minmax_scale.txt")
    q, s = oracle.quantize_row_f32(g["values"])
    S = max(abs(g["min_val"][0]), abs(g["max_val"][0])) / 127
    assert abs(s - S) <= ulp32(S) / 2
    assert q[0] == g["code_of_min"][0]
    assert q.max() <= 127 and q.min() >= -127


# ----------------------------------------------------------------- quantization invariants


def test_round_half_even_ties():
    # amax = 127 gives s = 1 exactly, so y/s hits exact .5 ties
    y = np.array([2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 127.0], dtype=np.float32)
    q, s = oracle.quantize_row_f32(y)
    assert s == 1.0
    assert list(q) == [2, 4, -2, -4, 0, 0, 2, 127]


def test_zero_row():
    q, s = oracle.quantize_row_f32(np.zeros(64, dtype=np.float32))
    assert s == 0.0 and not q.any()


@pytest.mark.parametrize("seed", range(4))
def test_quantize_invariants(seed):
    x = synth.activation(64, 512, seed)
    sinv = (1.0 / (1.0 + np.abs(synth.normal_bf16((512,), seed + 1).view(np.int16))
                   .astype(np.float32) / 3e4)).astype(np.float32)
    for sv in (None, sinv):
        q, s = oracle.quantize_rows(x, sv)
        y = oracle.bf16_to_f32(x).astype(np.float64)
        if sv is not None:
            y = (oracle.bf16_to_f32(x) * sv).astype(np.float64)  # binary32 product
        amax = np.abs(y).max(axis=1)
        for m in range(y.shape[0]):
            # scale: the binary32 nearest to amax/127
            exact = Fraction(float(amax[m])) / 127
            assert abs(Fraction(float(s[m])) - exact) <= Fraction(ulp32(s[m])) / 2
            assert np.abs(q[m]).max() == 127
            j = int(np.argmax(np.abs(y[m])))
            assert abs(int(q[m, j])) == 127 and np.sign(q[m, j]) == np.sign(y[m, j])
            err = np.abs(q[m].astype(np.float64) * float(s[m]) - y[m])
            assert (err <= float(s[m]) * (0.5 + 2.0 ** -16)).all()


def test_quantize_rows_sinv_is_a_division_by_s():
    # With sinv = 1/s the quantized row represents X diag(1/s): doubling a channel's s halves
    # that channel's code (up to rounding).
    x = synth.activation(4, 256, 3, outliers=0)
    sinv = np.ones(256, dtype=np.float32)
    sinv[::2] = 0.5
    q1, s1 = oracle.quantize_rows(x, None)
    q2, s2 = oracle.quantize_rows(x, sinv)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    rec = q2.astype(np.float64) * s2[:, None]
    assert np.all(np.abs(rec[:, ::2] - 0.5 * xf[:, ::2]) <= s2[:, None] * 0.5001)
    assert np.all(np.abs(rec[:, 1::2] - xf[:, 1::2]) <= s2[:, None] * 0.5001)


# ----------------------------------------------------------------- bf16 conversion


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * 10,
        np.array([1.0, 1.00390625, 1.001953125, 1.005859375, -1.001953125, 3.4e38, 1e-40,
                  0.0, -0.0, np.inf, -np.inf], dtype=np.float32)])
    ours = oracle.f32_to_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(oracle.bf16_to_f32(ours),
                          torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float()
                          .numpy())


# ----------------------------------------------------------------- RMSNorm


def test_rmsnorm_constant_rows():
    K = 256
    eps = 1e-5
    vals = [1.0, -3.0, 0.125, 17.5]
    x = synth.normal_bf16((len(vals), K), 0)
    xf = np.repeat(np.array(vals, dtype=np.float32)[:, None], K, axis=1)
    x = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    r = oracle.smooth_rmsnorm_quant(x, np.ones(K, np.float32), eps, want_y=True)
    for i, c in enumerate(vals):
        assert r["ms"][i] == f32(c * c)
        ref = c / math.sqrt(c * c + eps)
        assert abs(r["y"][i, 0] - ref) <= ulp32(ref)
        assert (np.abs(r["q"][i]) == 127).all()


@pytest.mark.parametrize("seed", range(3))
def test_rmsnorm_textbook_and_exact_mean(seed):
    M, K, eps = 24, 256, 1e-5
    x = synth.activation(M, K, seed)
    gam = synth.gamma(K, seed + 5)
    r = oracle.smooth_rmsnorm_quant(x, gam, eps, want_y=True)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    for m in range(M):
        exact = sum(Fraction(float(v)) ** 2 for v in xf[m]) / K
        ms_exact = round_fraction_to_f32(exact)
        if r["ambiguous"][m]:
            assert abs(r["ms"][m] - ms_exact) <= ulp32(ms_exact)
        else:
            assert r["ms"][m] == ms_exact
        rstd64 = 1.0 / math.sqrt(float(exact) + eps)
        ref = xf[m] * rstd64 * gam.astype(np.float64)
        assert np.all(np.abs(r["y"][m] - ref) <= 3 * np.spacing(np.abs(ref).astype(np.float32)))


def test_rmsnorm_residual_and_override():
    M, K, eps = 8, 128, 1e-5
    x = synth.activation(M, K, 11)
    res = synth.normal_bf16((M, K), 12)
    gam = synth.gamma(K, 13)
    r = oracle.smooth_rmsnorm_quant(x, gam, eps, residual=res)
    tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    tr = torch.from_numpy(res.view(np.int16)).view(torch.bfloat16)
    ref_h = (tx + tr).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["h"], ref_h)
    # a zero residual leaves x unchanged
    z = oracle.smooth_rmsnorm_quant(x, gam, eps, residual=np.zeros_like(x))
    assert np.array_equal(z["h"], x)
    plain = oracle.smooth_rmsnorm_quant(x, gam, eps)
    assert np.array_equal(z["q"], plain["q"]) and np.array_equal(z["s"], plain["s"])
    # forcing the mean of squares reproduces the unforced result
    f = oracle.smooth_rmsnorm_quant(x, gam, eps, ms_override=plain["ms"])
    assert np.array_equal(f["q"], plain["q"])
    # and scaling gamma by 2 leaves codes unchanged but doubles the scale
    d = oracle.smooth_rmsnorm_quant(x, gam * 2, eps)
    assert np.array_equal(d["q"], plain["q"]) and np.array_equal(d["s"], plain["s"] * 2)


# ----------------------------------------------------------------- exp / SiLU


def test_exp_against_binary64():
    xs = np.concatenate([np.linspace(-103.5, 88.7, 200001, dtype=np.float64),
                         np.linspace(-1, 1, 20001)]).astype(np.float32)
    worst = 0.0
    prev = -1.0
    for x in xs[:: 1]:
        v = oracle.exp(x)
        ref = math.exp(float(x))
        if ref < 2.0 ** -126:
            assert abs(v - ref) <= 2 * 2.0 ** -149
        elif ref > 3.4028234663852886e38:
            assert v == math.inf
        else:
            worst = max(worst, abs(v - ref) / ulp32(ref))
    assert worst <= 2.0
    assert oracle.exp(0.0) == 1.0
    assert oracle.exp(89.5) == math.inf and oracle.exp(-104.5) == 0.0
    sweep = [oracle.exp(x) for x in np.linspace(-30, 30, 5001, dtype=np.float32)]
    assert all(b >= a for a, b in zip(sweep, sweep[1:]))


def _rn32(q):
    """Round an exact rational to the nearest binary32 value, ties to even, with gradual
    underflow (quantum 2^-149) and overflow to infinity. Returns a Fraction or +-inf."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * quantum
    if v >= Fraction(2) ** 128:
        return math.inf if q > 0 else -math.inf
    return v if q > 0 else -v


def _exp_spec(x):
    """The binary32 exp exactly as the header writes it down, each operation evaluated in
    exact rational arithmetic and rounded once to binary32 (an fma rounds once): Cody-Waite
    reduction with k = rint(RN(x * RN(1/ln 2))), r = fma(-k, ln2_hi, x), r = fma(-k, ln2_lo, r)
    (ln2_hi = ln 2 to 16 significant bits, ln2_lo = RN(ln 2 - ln2_hi)); the degree-7 Taylor
    polynomial with coefficients RN(1/i!) by Horner's rule in fma; then times 2^(k/2) and
    2^(k - k/2) (k/2 truncated toward zero); x > 89 -> +inf, x < -104 -> +0."""
    import decimal
    ctx = decimal.Context(prec=60)
    ln2_dec = ctx.ln(decimal.Decimal(2))
    ln2 = Fraction(ln2_dec)
    x = Fraction(float(x))
    if x > 89:
        return math.inf
    if x < -104:
        return 0.0
    log2e = _rn32(Fraction(ctx.divide(decimal.Decimal(1), ln2_dec)))
    ln2_hi = Fraction(math.floor(ln2 * 2 ** 16), 2 ** 16)  # bit 17 of ln 2 is 0: floor = RN
    ln2_lo = _rn32(ln2 - ln2_hi)
    k = round(_rn32(x * log2e))  # Fraction.__round__ rounds half to even, as rint does
    r = _rn32(-k * ln2_hi + x)
    r = _rn32(-k * ln2_lo + r)
    c = [_rn32(Fraction(1, math.factorial(i))) for i in range(8)]
    p = c[7]
    for i in range(6, -1, -1):
        p = _rn32(p * r + c[i])
    k1 = int(k / 2) if k >= 0 else -int(-k / 2)
    k2 = k - k1
    v = _rn32(p * Fraction(2) ** k1)
    if v in (math.inf, -math.inf):
        return v
    v = _rn32(v * Fraction(2) ** k2)
    return float(v)


def test_exp_bits_match_an_exact_evaluation_of_its_written_definition():
    # Pins every bit of the oracle's exp (and so of the SiLU the GPU must reproduce) to the
    # header's written definition, evaluated independently with exact rationals: a dropped
    # Horner term, a wrong constant or a different scaling split changes many of these bits.
    rng = np.random.default_rng(11)
    f32 = np.float32
    ln2 = math.log(2.0)
    xs = [f32(0.0), f32(-0.0), f32(89.0), np.nextafter(f32(89.0), f32(100)), f32(-104.0),
          np.nextafter(f32(-104.0), f32(-200)), f32(88.72283), f32(88.7228394),
          f32(-87.33654), f32(-87.336548), f32(-103.278931), f32(-103.97), f32(1e-8),
          f32(-1e-8), f32(2.0 ** -30), f32(0.5), f32(-0.5), f32(1.0), f32(-1.0)]
    for j in range(-150, 129, 3):  # arguments where k changes, and their neighbours
        t = f32((j + 0.5) * ln2)
        xs += [t, np.nextafter(t, f32(200)), np.nextafter(t, f32(-200))]
    xs += list(np.linspace(-104, 89, 1200, dtype=np.float32))
    xs += list(rng.uniform(-104, 89, 1500).astype(np.float32))
    xs += list(rng.uniform(-1, 1, 500).astype(np.float32))
    mismatches = []
    for x in xs:
        got = f32(oracle.exp(x))
        want = f32(_exp_spec(x))
        if got.view(np.uint32) != want.view(np.uint32):
            mismatches.append((float(x), float(got), float(want)))
    assert not mismatches, mismatches[:5]


def test_silu_special_values_and_accuracy():
    assert oracle.silu(0.0) == 0.0
    for g in (20.0, 50.0, 88.0, 100.0):
        assert oracle.silu(g) == g
    assert oracle.silu(-100.0) == 0.0 and math.copysign(1, oracle.silu(-100.0)) == -1
    for g in np.linspace(-20, 20, 4001, dtype=np.float32):
        ref = float(g) / (1.0 + math.exp(-float(g)))
        if ref == 0.0:
            continue
        assert abs(oracle.silu(g) - ref) <= 4 * ulp32(ref)


def test_silu_mul_quant_bound():
    M, I = 6, 384
    gu = synth.normal_bf16((M, 2 * I), 21, std=3.0)
    q, s = oracle.silu_mul_quant(gu)
    gf = oracle.bf16_to_f32(gu).astype(np.float64)
    g, u = gf[:, :I], gf[:, I:]
    a = g / (1.0 + np.exp(-g)) * u
    assert (np.abs(q).max(axis=1) == 127).all()
    err = np.abs(q * s[:, None].astype(np.float64) - a)
    assert (err <= s[:, None] * 0.5 + np.abs(a) * 8 * F32_EPS).all()
    # swapping the gate and up halves changes the result (operands are not symmetric)
    q2, _ = oracle.silu_mul_quant(np.concatenate([gu[:, I:], gu[:, :I]], axis=1))
    assert not np.array_equal(q, q2)


# ----------------------------------------------------------------- GEMM + dequant


def test_gemm_brute_force_tiny():
    rng = np.random.default_rng(5)
    for (M, N, K) in [(1, 1, 1), (2, 3, 5), (3, 8, 8), (8, 8, 7), (5, 2, 8)]:
        xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
        xq[0, :] = 127
        wq[-1, :] = -127
        st = synth.scales(M, 1)
        sc = synth.scales(N, 2)
        y, acc = oracle.gemm_dequant(xq, st, wq, sc)
        for m in range(M):
            for n in range(N):
                a = 0
                for k in range(K):
                    a += int(xq[m, k]) * int(wq[n, k])
                assert acc[m, n] == a
        assert acc[0, N - 1] == -127 * 127 * K


def test_gemm_fp64_and_extreme_magnitude():
    xq = synth.int8_codes((16, 3000), 7)
    wq = synth.int8_codes((24, 3000), 8)
    y, acc = oracle.gemm_dequant(xq, np.ones(16, np.float32), wq, np.ones(24, np.float32))
    ref = xq.astype(np.float64) @ wq.astype(np.float64).T
    assert np.array_equal(acc.astype(np.float64), ref)
    assert acc[0, 0] == 127 * 127 * 3000 and acc[0, 0] > 2 ** 24  # int->float rounds
    # transposing the weight is caught
    assert not np.array_equal(acc, (xq.astype(np.float64) @ wq[::-1].astype(np.float64).T))


def test_dequant_rounding():
    rng = np.random.default_rng(9)
    acc = rng.integers(-(2 ** 30), 2 ** 30, 4000).astype(np.int32)
    st = synth.scales(4000, 3)
    sc = synth.scales(4000, 4)
    ours = np.array([oracle.dequant(a, s, c) for a, s, c in zip(acc, st, sc)], np.uint16)
    t = (torch.from_numpy(acc).float() * torch.from_numpy(st)) * torch.from_numpy(sc)
    ref = t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    exact = acc.astype(np.float64) * st.astype(np.float64) * sc.astype(np.float64)
    got = oracle.bf16_to_f32(ours).astype(np.float64)
    assert np.all(np.abs(got - exact) <= np.abs(exact) * 2.0 ** -8)
    assert oracle.dequant(12345, 0.0, 1.0) == 0


def test_gemm_sampled_matches_full():
    xq = synth.int8_codes((40, 512), 1)
    wq = synth.int8_codes((72, 512), 2)
    st, sc = synth.scales(40, 3), synth.scales(72, 4)
    y, acc = oracle.gemm_dequant(xq, st, wq, sc)
    ms = np.array([0, 39, 5, 17])
    ns = np.array([71, 0, 33, 8])
    ys, accs = oracle.gemm_dequant_sampled(xq, st, wq, sc, ms, ns)
    assert np.array_equal(ys, y[ms, ns]) and np.array_equal(accs, acc[ms, ns])


# ----------------------------------------------------------------- SmoothQuant prep


def test_column_absmax():
    a = np.random.default_rng(1).standard_normal((33, 17)).astype(np.float32)
    assert np.array_equal(oracle.column_absmax_f32(a), np.abs(a).max(axis=0))
    w = synth.weight(19, 40, 2)
    assert np.array_equal(oracle.column_absmax_bf16(w),
                          np.abs(oracle.bf16_to_f32(w)).max(axis=0))


@pytest.mark.parametrize("alpha", [0.5, 0.8])
def test_smoothing_factor_balances_maxima(alpha):
    # SmoothQuant migrates difficulty: after smoothing, max|X_j| / s_j and max|W_j| * s_j
    # stand in the ratio (a_j w_j)^(1 - 2 alpha); at alpha = 0.5 they are equal.
    rng = np.random.default_rng(2)
    a = (np.abs(rng.standard_normal(300)) * 10 + 1e-3).astype(np.float32)
    w = (np.abs(rng.standard_normal(300)) * 0.05 + 1e-4).astype(np.float32)
    s = oracle.smoothing_factors(a, w, alpha).astype(np.float64)
    lhs = (a / s) / (w * s)
    rhs = (a.astype(np.float64) * w) ** (1 - 2 * alpha)
    assert np.allclose(lhs, rhs, rtol=4e-7)
    # outlier channels get large factors (the page: proportional to the outlier's severity)
    if alpha == 0.5:
        assert s[np.argmax(a / w)] == s.max()
    assert s[np.argmax(a)] > np.median(s)
    z = oracle.smoothing_factors(np.array([0.0, 2.0], np.float32),
                                 np.array([1.0, 0.0], np.float32), alpha)
    assert list(z) == [1.0, 1.0]


def test_smoothquant_identity():
    # (X diag(1/s)) (diag(s) W^T) = X W^T to binary32 rounding of the folded operands
    M, N, K = 8, 12, 256
    x = synth.activation(M, K, 4)
    w = synth.weight(N, K, 5)
    xf = oracle.bf16_to_f32(x)
    s = oracle.smoothing_factors(oracle.column_absmax_f32(xf), oracle.column_absmax_bf16(w),
                                 0.5)
    _, sinv = oracle.fold_gamma(np.ones(K, np.float32), s)
    ws = oracle.smooth_weight(w, s).astype(np.float64)
    xs = (xf * sinv).astype(np.float64)
    wf = oracle.bf16_to_f32(w).astype(np.float64)
    lhs = xs @ ws.T
    ref = xf.astype(np.float64) @ wf.T
    bound = 4 * 2.0 ** -24 * (np.abs(xf).astype(np.float64) @ np.abs(wf).T)
    assert np.all(np.abs(lhs - ref) <= bound)
    # smoothing really moved the outliers: the per-channel maxima of X' are flatter
    assert np.abs(xs).max(axis=0).max() / np.median(np.abs(xs).max(axis=0)) < \
        np.abs(xf).max(axis=0).max() / np.median(np.abs(xf).max(axis=0))


def test_rtn_weights_are_rowwise_quant_of_smoothed_weight():
    w = synth.weight(16, 256, 6)
    s = (1.0 + np.arange(256, dtype=np.float32) / 256).astype(np.float32)
    wq, s_ch = oracle.rtn_weights(w, s)
    ws = oracle.smooth_weight(w, s).astype(np.float64)
    assert (np.abs(wq).max(axis=1) == 127).all()
    err = np.abs(wq * s_ch[:, None].astype(np.float64) - ws)
    assert (err <= s_ch[:, None] * (0.5 + 2.0 ** -16)).all()
    for n in range(16):
        exact = Fraction(float(np.abs(ws[n]).max())) / 127
        assert abs(Fraction(float(s_ch[n])) - exact) <= Fraction(ulp32(s_ch[n])) / 2


# ----------------------------------------------------------------- static per-tensor scale


def _bf16_bits(xf):
    return torch.from_numpy(np.asarray(xf, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_static_minmax_calibration_worked_example(golden):
    # the page's calibration set: S = max(|min|, |max|) / 127 and the most negative value
    # codes to -127 with that fixed scale
    g = golden("p3_minmax_scale.txt")
    S = oracle.minmax_scale(np.array(g["values"], np.float32))
    ref = Fraction(max(abs(g["min_val"][0]), abs(g["max_val"][0]))) / 127
    assert float(S) == round_fraction_to_f32(ref)
    q = oracle.quantize_rows_static(_bf16_bits([g["values"]]), S)
    assert q[0, 0] == g["code_of_min"][0]
    assert q.max() <= 127 and q.min() >= -127


def test_static_reduces_to_dynamic_with_the_rows_own_scale():
    # with S equal to a row's own dynamic scale, static quantization is per-token dynamic
    # quantization of that row (including its smoothing)
    x = synth.activation(6, 512, seed=3)
    sinv = (1.0 / synth.gamma(512, 4)).astype(np.float32)
    q_dyn, s_dyn = oracle.quantize_rows(x, sinv)
    for m in range(6):
        q_st = oracle.quantize_rows_static(x[m:m + 1], s_dyn[m], sinv)
        assert np.array_equal(q_st[0], q_dyn[m])


def test_static_exact_multiples_ties_and_saturation():
    # S = 2^-4: y = k S is exact, (k + 1/2) S is an exact tie (half to even), and values
    # past 127 S saturate
    S = np.float32(0.0625)
    k = np.arange(-140, 141)
    y = np.concatenate([k * 0.0625, (np.arange(-20, 20) + 0.5) * 0.0625]).astype(np.float32)
    q = oracle.quantize_rows_static(_bf16_bits([y]), S)[0]
    expect_k = np.clip(k, -127, 127)
    # j + 1/2 lies between j and j + 1: the even one of the two
    expect_h = np.array([j if j % 2 == 0 else j + 1 for j in range(-20, 20)])
    assert np.array_equal(q[:len(k)], expect_k)
    assert np.array_equal(q[len(k):], expect_h)


def test_static_rejects_nonpositive_scale():
    x = _bf16_bits([[1.0, 2.0]])
    for bad in (0.0, -1.0):
        with pytest.raises(ValueError):
            oracle.quantize_rows_static(x, bad)


def test_silu_mul_is_what_silu_mul_quant_quantizes():
    gu = synth.normal_bf16((5, 2 * 96), seed=8, std=2.5)
    a = oracle.silu_mul(gu)
    g = oracle.bf16_to_f32(gu[:, :96])
    u = oracle.bf16_to_f32(gu[:, 96:])
    # element by element: the scalar SiLU (pinned above) times up, one binary32 product
    for m in range(5):
        for j in range(0, 96, 7):
            assert a[m, j] == np.float32(np.float32(oracle.silu(float(g[m, j]))) * u[m, j])
    q, s = oracle.silu_mul_quant(gu)
    for m in range(5):
        q1, s1 = oracle.quantize_row_f32(a[m])
        assert s1 == s[m] and np.array_equal(q1, q[m])
