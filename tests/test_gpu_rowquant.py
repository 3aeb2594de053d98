"""Parity of the per-token quantization kernels with the oracle, through the C ABI:
int8 codes, fp32 scales and bf16 residual sums bit-exact, on shapes spanning one vector per
thread up to the largest rows, ragged rows and zero rows."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import synth
from helpers import (assert_rms_rows_match, bf16_out, dev, dev_bf16, f32_out, host, host_bf16,
                     i8_out)

pytestmark = pytest.mark.gpu

ROW_SHAPES = [(1, 16), (3, 48), (16, 256), (37, 4096), (5, 8192), (64, 14336), (3, 28672),
              (2, 32768), (300, 4096), (7, 4112)]


def _sinv(K, seed):
    g = synth.gamma(K, seed)  # positive values around 1
    return (1.0 / np.abs(g)).astype(np.float32)


@pytest.mark.parametrize("M,K", ROW_SHAPES)
@pytest.mark.parametrize("smooth", [False, True])
def test_quantize_rows_bit_exact(M, K, smooth):
    x = synth.activation(M, K, seed=M * 7 + K)
    sinv = _sinv(K, K) if smooth else None
    q_ref, s_ref = oracle.quantize_rows(x, sinv)
    q, cq = i8_out((M, K))
    s, cs = f32_out((M,))
    w8.w8a8_quantize_rows(dev_bf16(x), None if sinv is None else dev(sinv), q=q, s_tok=s)
    torch.cuda.synchronize()
    cq(); cs()
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)


def test_quantize_rows_zero_and_tie_rows():
    K = 64
    x = np.zeros((3, K), dtype=np.float32)
    x[1, :8] = [2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 127.0]  # s = 1: exact .5 ties
    x[2, 5] = -7.0
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q_ref, s_ref = oracle.quantize_rows(xb)
    q, s = w8.w8a8_quantize_rows(dev_bf16(xb))
    assert np.array_equal(host(s), s_ref) and np.array_equal(host(q), q_ref)
    assert host(s)[0] == 0 and not host(q)[0].any()
    assert list(host(q)[1, :8]) == [2, 4, -2, -4, 0, 0, 2, 127]


@pytest.mark.parametrize("M,K", [(1, 16), (7, 256), (33, 4096), (20, 8192), (3, 48), (129, 4096),
                                 (2, 28672)])
@pytest.mark.parametrize("with_residual", [False, True])
def test_smooth_rmsnorm_quant_bit_exact(M, K, with_residual):
    x = synth.activation(M, K, seed=3 * M + K)
    gam = synth.gamma(K, seed=K + 1)
    s_fac = _sinv(K, K + 2)  # any positive smoothing factors
    gf, _ = oracle.fold_gamma(gam, s_fac)
    res = synth.normal_bf16((M, K), seed=M + 5) if with_residual else None
    eps = 1e-5
    q, cq = i8_out((M, K))
    s, cs = f32_out((M,))
    if with_residual:
        h, ch = bf16_out((M, K))
        w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gf), eps, residual=dev_bf16(res), h_out=h,
                                     q=q, s_tok=s)
    else:
        w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gf), eps, q=q, s_tok=s)
    torch.cuda.synchronize()
    cq(); cs()
    ref, _ = assert_rms_rows_match(host(q), host(s), x, gf, eps, residual=res)
    if with_residual:
        ch()
        assert np.array_equal(host_bf16(h), ref["h"])


def test_smooth_rmsnorm_h_out_may_alias_residual():
    M, K = 9, 512
    x = synth.activation(M, K, 1)
    res = synth.normal_bf16((M, K), 2)
    gf = synth.gamma(K, 3)
    ref = oracle.smooth_rmsnorm_quant(x, gf, 1e-5, residual=res)
    r = dev_bf16(res)
    q, s, h = w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gf), 1e-5, residual=r, h_out=r)
    assert np.array_equal(host_bf16(h), ref["h"])
    assert_rms_rows_match(host(q), host(s), x, gf, 1e-5, residual=res, ref=ref)


@pytest.mark.parametrize("M,I", [(1, 16), (9, 256), (33, 14336), (4, 28672), (130, 4096),
                                 (2, 14352)])
def test_silu_mul_quant_bit_exact(M, I):
    gu = synth.normal_bf16((M, 2 * I), seed=M + I, std=2.5)
    if M > 1:  # a row reaching the exp overflow/underflow ranges
        gu[1, :8] = synth.normal_bf16((1, 8), 1)[0]
        vals = np.array([95.0, -95.0, 88.5, -88.5, 104.5, -104.5, 0.0, -0.0], np.float32)
        gu[1, :8] = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy() \
            .view(np.uint16)
    q_ref, s_ref = oracle.silu_mul_quant(gu)
    q, cq = i8_out((M, I))
    s, cs = f32_out((M,))
    w8.w8a8_silu_mul_quant(dev_bf16(gu), q=q, s_tok=s)
    torch.cuda.synchronize()
    cq(); cs()
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)


def test_weight_rtn_through_quantize_rows():
    # offline weight prep: quantize_rows(W, s) is the per-output-channel RTN of diag(s)-smoothed W
    N, K = 96, 4096
    w = synth.weight(N, K, 9)
    s_fac = (1.0 / _sinv(K, 10)).astype(np.float32)
    wq_ref, sch_ref = oracle.rtn_weights(w, s_fac)
    wq, sch = w8.w8a8_quantize_rows(dev_bf16(w), dev(s_fac))
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sch), sch_ref)


def test_device_status_clean():
    assert w8.w8a8_device_status(reset=True) == 0


def test_quantize_near_half_integer_quotients():
    # x holds j + 0.5 (j = 0..126) and 127, so with sinv near 1 every y / s lands within a few
    # ulps of a half-integer: the product-with-reciprocal shortcut must defer to the exact
    # quotient there, and ties must go to even
    K = 256
    base = np.concatenate([np.arange(127) + 0.5, [127.0], -(np.arange(127) + 0.5), [-127.0]])
    rows = []
    for i in range(64):
        rows.append(np.roll(base, i))
    xf = np.stack(rows).astype(np.float32)
    xb = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    rng = np.random.default_rng(0)
    for trial in range(4):
        sinv = (1.0 + (rng.integers(-8, 9, K) * 2.0 ** -23)).astype(np.float32)
        if trial == 0:
            sinv[:] = 1.0
        q_ref, s_ref = oracle.quantize_rows(xb, sinv)
        q, s = w8.w8a8_quantize_rows(dev_bf16(xb), dev(sinv))
        assert np.array_equal(host(s), s_ref)
        assert np.array_equal(host(q), q_ref)


# Row counts above the persistent grid (resident CTAs on the device), so that every CTA
# loops over several rows and, for blocks of up to 512 threads, prefetches the next row.
@pytest.mark.parametrize("M,K", [(5000, 256), (1500, 4096), (700, 28672)])
def test_quantize_rows_persistent_loop(M, K):
    x = synth.activation(M, K, seed=M + K + 17)
    sinv = _sinv(K, K + 3)
    q_ref, s_ref = oracle.quantize_rows(x, sinv)
    q, s = w8.w8a8_quantize_rows(dev_bf16(x), dev(sinv))
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)


@pytest.mark.parametrize("M,K", [(5000, 256), (1500, 4096), (600, 8192), (300, 28672)])
@pytest.mark.parametrize("with_residual", [False, True])
def test_smooth_rmsnorm_quant_persistent_loop(M, K, with_residual):
    x = synth.activation(M, K, seed=2 * M + K)
    gf = synth.gamma(K, seed=K + 7)
    res = synth.normal_bf16((M, K), seed=M + 9) if with_residual else None
    if with_residual:
        q, s, h = w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gf), 1e-5, residual=dev_bf16(res),
                                               h_out=torch.empty(M, K, dtype=torch.bfloat16,
                                                                 device="cuda"))
    else:
        q, s = w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gf), 1e-5)
    ref, _ = assert_rms_rows_match(host(q), host(s), x, gf, 1e-5, residual=res)
    if with_residual:
        assert np.array_equal(host_bf16(h), ref["h"])


@pytest.mark.parametrize("M,K", [(3, 4096), (600, 4096), (5, 8192), (300, 16384)])
@pytest.mark.parametrize("with_residual", [False, True])
def test_smooth_rmsnorm_quant_same_in_every_overlap_mode(M, K, with_residual):
    """Overlap mode 2 reads gamma' before the dependency wait (into registers for rows of up
    to 4096 values, into L2 for longer rows): the results are those of modes 0 and 1."""
    x = dev_bf16(synth.activation(M, K, seed=M + K))
    gf = dev(synth.gamma(K, seed=K + 3))
    res = dev_bf16(synth.normal_bf16((M, K), seed=M + 5)) if with_residual else None
    prev = w8.w8a8_get_overlap()
    out = {}
    try:
        for mode in (0, 1, 2):
            w8.w8a8_set_overlap(mode)
            h = torch.empty(M, K, dtype=torch.bfloat16, device="cuda") if with_residual else None
            r = w8.w8a8_smooth_rmsnorm_quant(x, gf, 1e-5, residual=res, h_out=h)
            torch.cuda.synchronize()
            out[mode] = [host(t) if t.dtype != torch.bfloat16 else host_bf16(t) for t in r]
    finally:
        w8.w8a8_set_overlap(prev)
    for mode in (1, 2):
        for a, b in zip(out[0], out[mode]):
            assert np.array_equal(a, b), f"overlap mode {mode}"
    ref, _ = assert_rms_rows_match(out[2][0], out[2][1], synth.activation(M, K, seed=M + K),
                                   synth.gamma(K, seed=K + 3), 1e-5,
                                   residual=synth.normal_bf16((M, K), seed=M + 5)
                                   if with_residual else None)


@pytest.mark.parametrize("M,I", [(5000, 128), (700, 14336), (300, 28672)])
def test_silu_mul_quant_persistent_loop(M, I):
    gu = synth.normal_bf16((M, 2 * I), seed=M + I + 5, std=2.5)
    q_ref, s_ref = oracle.silu_mul_quant(gu)
    q, s = w8.w8a8_silu_mul_quant(dev_bf16(gu))
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)


def test_quantize_tiny_scales_take_exact_quotient():
    # rows whose absmax is so small that the scale is below 2^-100 (the reciprocal would
    # leave the binary32 range) are quantized through the exact quotient
    K = 256
    rng = np.random.default_rng(5)
    rows = []
    for mag in (1e-38, 3e-35, 1e-30, 1e-28, 1.0):
        rows.append(rng.standard_normal(K) * mag)
    xf = np.stack(rows).astype(np.float32)
    xb = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q_ref, s_ref = oracle.quantize_rows(xb)
    q, s = w8.w8a8_quantize_rows(dev_bf16(xb))
    assert np.array_equal(host(s), s_ref)
    assert np.array_equal(host(q), q_ref)
    assert (s_ref[:3] < 2.0 ** -100).all() and s_ref[3] > 2.0 ** -100


@pytest.mark.parametrize("M,K", [(1, 16), (37, 4096), (300, 4112), (3000, 4096), (5, 28672)])
@pytest.mark.parametrize("smooth", [False, True])
def test_quantize_rows_static_bit_exact(M, K, smooth):
    # the scale is calibrated on a different batch, so some values of x lie beyond it and
    # saturate; the near-half-integer and exact-quotient paths are exercised by the data
    x = synth.activation(M, K, seed=M + 3 * K)
    cal = synth.activation(64, K, seed=K + 11)
    sinv = _sinv(K, K + 5) if smooth else None
    calf = oracle.bf16_to_f32(cal) * (sinv if smooth else 1.0)
    S = oracle.minmax_scale(calf.astype(np.float32)) * np.float32(0.5)
    q_ref = oracle.quantize_rows_static(x, S, sinv)
    q, s = w8.w8a8_quantize_rows_static(dev_bf16(x), float(S), None if sinv is None else dev(sinv))
    assert np.array_equal(host(q), q_ref)
    assert (host(s) == S).all()
    if M * K >= 4096:
        assert (np.abs(q_ref) == 127).any()  # saturation happened


def test_quantize_rows_static_tiny_and_equal_to_dynamic():
    # a scale below 2^-100 takes the exact quotient; with a row's own dynamic scale the codes
    # are the dynamic codes
    K = 256
    x = synth.activation(4, K, 21)
    q_dyn, s_dyn = oracle.quantize_rows(x)
    for m in range(4):
        q, _ = w8.w8a8_quantize_rows_static(dev_bf16(x[m:m + 1]), float(s_dyn[m]))
        assert np.array_equal(host(q)[0], q_dyn[m])
    tiny = (synth.activation(2, K, 22).view(np.uint16) & 0x807F) | 0x0080  # |x| ~ 2^-126
    S = np.float32(2.0 ** -132)  # subnormal: |x| / S in [64, 128), the largest saturate
    q, _ = w8.w8a8_quantize_rows_static(dev_bf16(tiny), float(S))
    q_ref = oracle.quantize_rows_static(tiny, S)
    assert np.array_equal(host(q), q_ref)
    assert (np.abs(q_ref) >= 64).all() and (np.abs(q_ref) == 127).any()


def test_static_scale_calibration_matches_oracle():
    from int8_w8a8_quantized_smoothed_b200 import prep
    cal = synth.activation(128, 4096, 31)
    sinv = _sinv(4096, 32)
    S = prep.static_activation_scale(dev_bf16(cal), dev(sinv))
    ref = oracle.minmax_scale((oracle.bf16_to_f32(cal) * sinv).astype(np.float32))
    assert np.float32(S) == ref


def test_wait_timeout_reports_status_and_context_stays_usable():
    # a wait that nothing satisfies gives up after its limit, raises the status word and the
    # kernel returns; afterwards the context runs kernels normally
    assert w8.w8a8_device_status(reset=True) == 0
    w8.w8a8_selftest_wait_timeout(2_000_000)  # 2 ms
    assert w8.w8a8_device_status(reset=True) == -6  # W8A8_ERR_TIMEOUT
    assert w8.w8a8_device_status(reset=False) == 0
    x = synth.activation(4, 256, 3)
    q_ref, s_ref = oracle.quantize_rows(x)
    q, s = w8.w8a8_quantize_rows(dev_bf16(x))
    assert np.array_equal(host(q), q_ref) and np.array_equal(host(s), s_ref)
    with pytest.raises(w8.W8A8Error):
        w8.w8a8_selftest_wait_timeout(10)  # below the allowed range


def test_stream_status_reports_timeout_of_that_streams_kernel():
    # w8a8_last_device_status waits for one stream only and reads the device word without
    # clearing it
    assert w8.w8a8_device_status(reset=True) == 0
    s = torch.cuda.Stream()
    assert w8.w8a8_last_device_status(s) == 0
    w8.w8a8_selftest_wait_timeout(2_000_000, stream=s)
    assert w8.w8a8_last_device_status(s) == -6
    assert w8.w8a8_last_device_status(s) == -6  # not cleared by reading
    assert w8.w8a8_device_status(reset=True) == -6
    assert w8.w8a8_last_device_status(s) == 0
    assert w8.w8a8_last_device_status() == 0
