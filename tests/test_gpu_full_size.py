"""Parity at the workloads' full sizes, in the launch configuration the benchmark times
(automatic kernel choice, default workspace): the Llama-3.1-8B decode set (M = 1, 8, 32, 64),
the prefill set (M = 2048, 8192), and the Llama-3.1-70B set (M = 16, 4096). The oracle
checks a seeded sample of outputs one by one (first/last rows and channels included); the
row kernels are checked on sampled rows."""
import zlib

import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import synth
from helpers import assert_rms_rows_match, dev, dev_bf16, host, host_bf16

pytestmark = pytest.mark.gpu

LLAMA8B = dict(H=4096, I=14336, QKV=6144)
LLAMA70B = dict(H=8192, I=28672, QKV=10240)


def projections(cfg):
    H, I, QKV = cfg["H"], cfg["I"], cfg["QKV"]
    return [("qkv", QKV, H), ("o", H, H), ("gate_up", 2 * I, H), ("down", H, I)]


def _seed(name, M):
    return zlib.crc32(f"{name}/{M}".encode()) % 1000


def _sample_pairs(M, N, seed, count=1500):
    rng = np.random.default_rng(seed)
    ms = np.concatenate([[0, M - 1, 0, M - 1], rng.integers(0, M, count)])
    ns = np.concatenate([[0, N - 1, N - 1, 0], rng.integers(0, N, count)])
    return ms, ns


_WCACHE = {}


def _weight_codes(N, K, seed):
    key = (N, K, seed)
    if key not in _WCACHE:
        _WCACHE.clear()
        _WCACHE[key] = synth.int8_codes((N, K), seed, extremes=False)
    return _WCACHE[key]


def _check_gemm(M, N, K, seed, wseed):
    xq = synth.int8_codes((M, K), seed)
    wq = _weight_codes(N, K, wseed)
    st = synth.scales(M, seed + 2, 1e-3, 0.5)
    sc = synth.scales(N, seed + 3, 1e-4, 2e-2)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = w8.w8a8_gemm_dequant(dev(xq), dev(st), dev(wq), dev(sc), acc_out=acc)
    y2 = w8.w8a8_gemm_dequant(dev(xq), dev(st), dev(wq), dev(sc))  # no check-mode output
    torch.cuda.synchronize()
    ms, ns = _sample_pairs(M, N, seed)
    y_ref, acc_ref = oracle.gemm_dequant_sampled(xq, st, wq, sc, ms, ns)
    yh, ah = host_bf16(y), host(acc)
    assert np.array_equal(ah[ms, ns], acc_ref)
    assert np.array_equal(yh[ms, ns], y_ref)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M", [1, 8, 32, 64])
@pytest.mark.parametrize("name,N,K", projections(LLAMA8B))
def test_llama8b_decode_gemm(M, name, N, K):
    _check_gemm(M, N, K, _seed(name, M), _seed(name, 0))


@pytest.mark.parametrize("M", [2048, 8192])
@pytest.mark.parametrize("name,N,K", projections(LLAMA8B))
def test_llama8b_prefill_gemm(M, name, N, K):
    _check_gemm(M, N, K, _seed(name, M) + 1, _seed(name, 0))


@pytest.mark.parametrize("M", [16, 4096])
@pytest.mark.parametrize("name,N,K", projections(LLAMA70B))
def test_llama70b_gemm(M, name, N, K):
    _check_gemm(M, N, K, _seed(name, M) + 2, _seed(name, 1))


@pytest.mark.parametrize("M,H,I", [(8192, 4096, 14336), (4096, 8192, 28672), (64, 4096, 14336)])
def test_row_kernels_full_size_sampled_rows(M, H, I):
    rows = synth.row_sample(M, 3, count=48)
    x = synth.activation(M, H, 1)
    res = synth.normal_bf16((M, H), 2)
    gam = synth.gamma(H, 3)
    sinv = (1.0 / synth.gamma(H, 4)).astype(np.float32)
    q, s, h = w8.w8a8_smooth_rmsnorm_quant(dev_bf16(x), dev(gam), 1e-5, residual=dev_bf16(res))
    ref, _ = assert_rms_rows_match(host(q)[rows], host(s)[rows], x[rows], gam, 1e-5,
                                   residual=res[rows])
    assert np.array_equal(host_bf16(h)[rows], ref["h"])
    q, s = w8.w8a8_quantize_rows(dev_bf16(x), dev(sinv))
    q_ref, s_ref = oracle.quantize_rows(x[rows], sinv)
    assert np.array_equal(host(q)[rows], q_ref) and np.array_equal(host(s)[rows], s_ref)
    gu = synth.normal_bf16((M, 2 * I), 5, std=2.0)
    q, s = w8.w8a8_silu_mul_quant(dev_bf16(gu))
    q_ref, s_ref = oracle.silu_mul_quant(gu[rows])
    assert np.array_equal(host(q)[rows], q_ref) and np.array_equal(host(s)[rows], s_ref)


# ------------------------------------------------------------------ FP8 (E4M3) at full size


def _fp8_codes(shape, seed):
    c = np.random.default_rng(seed).integers(0, 256, shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return c


def _dev_fp8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(w8.FP8)


def _check_gemm_fp8(M, N, K, seed, wseed):
    xq = _fp8_codes((M, K), seed)
    wq = _fp8_codes((N, K), wseed)
    st = synth.scales(M, seed + 2, 1e-3, 0.5)
    sc = synth.scales(N, seed + 3, 1e-4, 2e-2)
    acc = torch.empty((M, N), dtype=torch.float32, device="cuda")
    y = w8.w8a8_gemm_dequant_fp8(_dev_fp8(xq), dev(st), _dev_fp8(wq), dev(sc), acc_out=acc)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, M - 1], synth.row_sample(M, seed, count=6)]))
    _, acc_ref, absacc = oracle.gemm_fp8(xq[rows], st[rows], wq, sc)
    a = host(acc)[rows].astype(np.float64)
    assert (np.abs(a - acc_ref) <= (K + 16) * 2.0 ** -24 * absacc).all()
    # empirical guard (measured at most 14 units of 2^-24 * sum|products| on B200)
    assert (np.abs(a - acc_ref) <= 64 * 2.0 ** -24 * absacc).all()
    assert np.array_equal(host_bf16(y)[rows], oracle.dequant_f32acc(host(acc)[rows], st[rows], sc))


@pytest.mark.parametrize("M", [1, 64, 2048])
@pytest.mark.parametrize("name,N,K", projections(LLAMA8B))
def test_llama8b_gemm_fp8(M, name, N, K):
    _check_gemm_fp8(M, N, K, _seed(name, M) + 3, _seed(name, 2))


@pytest.mark.parametrize("M", [16, 4096])
@pytest.mark.parametrize("name,N,K", projections(LLAMA70B))
def test_llama70b_gemm_fp8(M, name, N, K):
    _check_gemm_fp8(M, N, K, _seed(name, M) + 4, _seed(name, 3))


@pytest.mark.parametrize("M,H,I", [(8192, 4096, 14336), (64, 4096, 14336)])
def test_row_kernels_fp8_full_size_sampled_rows(M, H, I):
    rows = synth.row_sample(M, 5, count=32)
    x = synth.activation(M, H, 11)
    res = synth.normal_bf16((M, H), 12)
    gam = synth.gamma(H, 13)
    q, s, h = w8.w8a8_smooth_rmsnorm_quant_fp8(dev_bf16(x), dev(gam), 1e-5,
                                               residual=dev_bf16(res))
    ref, _ = assert_rms_rows_match(q.view(torch.uint8).cpu().numpy()[rows], host(s)[rows],
                                   x[rows], gam, 1e-5, residual=res[rows],
                                   ref_fn=oracle.smooth_rmsnorm_quant_fp8)
    assert np.array_equal(host_bf16(h)[rows], ref["h"])
    gu = synth.normal_bf16((M, 2 * I), 15, std=2.0)
    q, s = w8.w8a8_silu_mul_quant_fp8(dev_bf16(gu))
    q_ref, s_ref = oracle.silu_mul_quant_fp8(gu[rows])
    assert np.array_equal(q.view(torch.uint8).cpu().numpy()[rows], q_ref)
    assert np.array_equal(host(s)[rows], s_ref)
