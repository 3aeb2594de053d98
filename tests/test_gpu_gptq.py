"""Parity of the GPU GPTQ with the oracle, through the C ABI.

The GPU applies the column updates in blocks of 64 (lazy batches), so its binary64 sums run in
another order than the oracle's column-by-column loop: U (the inverse-Hessian factor) is
compared within a relative 1e-9, the scales bit-exactly, and the codes step by step: the
oracle re-runs the GPTQ recurrence propagating the GPU's own codes and judges every one of
them against its own decision at that step; a code may differ only by one, across a rounding
tie within 1e-8 of a quantization step (the size of the sum-order effect, ~1e-12, with a wide
margin). At the full 8B size the factor is checked by its defining identity U H U^T = I and
the codes on sampled rows.
"""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import synth
from helpers import dev, dev_bf16, host

pytestmark = pytest.mark.gpu

TIE_TOL = 1e-8


def _calib(T, K, seed, rho=0.6):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, K)).astype(np.float32)
    mix = (np.eye(K) + rho * rng.standard_normal((K, K)) / np.sqrt(K)).astype(np.float32)
    x = z @ mix
    x[:, rng.choice(K, max(1, K // 100), replace=False)] *= 20.0
    return x.astype(np.float32)


def _run(N, K, T, seed, smooth=True, dead=()):
    w = synth.weight(N, K, seed)
    s = (1.0 / synth.gamma(K, seed + 1) ** 2).astype(np.float32) if smooth else None
    x = _calib(T, K, seed + 2)
    for j in dead:
        x[:, j] = 0.0
    wq, sch, u = w8.w8a8_gptq_quantize(dev_bf16(w), dev(x), None if s is None else dev(s),
                                       want_u=True)
    torch.cuda.synchronize()
    wf = oracle.smooth_weight(w, s) if s is not None else oracle.bf16_to_f32(w)
    return w, wf, x, host(wq), host(sch), host(u)


def _follow(wf, dead, U, q, rows=None):
    if rows is not None:
        wf, q = wf[rows], q[rows]
    f = oracle.gptq_quantize(wf, dead, U, q_follow=q, tie_tol=TIE_TOL)
    bad = np.argwhere(f["status"] == 2)
    assert len(bad) == 0, f"{len(bad)} codes are no GPTQ decision, first at {bad[:3]}"
    return f, int((f["status"] == 1).sum())


@pytest.mark.parametrize("N,K,T", [(96, 256, 512), (200, 512, 256), (64, 1024, 1024),
                                   (8, 64, 16),
                                   # ragged groups of column blocks: 4 + 1 and 4 + 3 blocks
                                   (33, 320, 128), (1, 448, 64), (130, 448, 300),
                                   # more rows than one wave of the four-lane quantize
                                   # kernel holds: the one-thread-per-row kernel
                                   (20000, 128, 64)])
def test_gptq_matches_oracle(N, K, T):
    w, wf, x, q, sch, u = _run(N, K, T, seed=N + K)
    r = oracle.gptq(wf, x, damp=0.01)
    assert np.array_equal(sch, r["s"])
    assert np.abs(u - r["U"]).max() <= 1e-9 * np.abs(r["U"]).max()
    assert np.array_equal(u, np.triu(u))
    f, ties = _follow(wf, r["dead"], r["U"], q)
    assert ties <= max(2, q.size // 100000)
    # a trajectory that never crossed a tie is the oracle's own
    if ties == 0:
        assert np.array_equal(q, r["q"])


def test_gptq_dead_channels_and_no_smoothing():
    w, wf, x, q, sch, u = _run(64, 256, 128, seed=3, smooth=False, dead=(0, 17, 255))
    r = oracle.gptq(wf, x, damp=0.01)
    assert r["dead"][[0, 17, 255]].all()
    assert (q[:, [0, 17, 255]] == 0).all()
    assert np.array_equal(sch, r["s"])
    _follow(wf, r["dead"], r["U"], q)


def test_gptq_beats_rtn_on_layer_output():
    N, K, T = 128, 512, 1024
    w, wf, x, q, sch, u = _run(N, K, T, seed=11)
    q_rtn, s_rtn = oracle.rtn_weights(w, (1.0 / synth.gamma(K, 12) ** 2).astype(np.float32))
    x64 = x.astype(np.float64)

    def err(qq, ss):
        return np.sum(((wf.astype(np.float64) - qq * ss[:, None].astype(np.float64)) @ x64.T) ** 2)
    assert np.array_equal(sch, s_rtn)
    assert err(q, sch) < 0.9 * err(q_rtn, s_rtn)


def test_gptq_full_size_qkv_8b():
    """Llama-3.1-8B qkv projection (6144 x 4096), 512 calibration tokens."""
    N, K, T = 6144, 4096, 512
    w, wf, x, q, sch, u = _run(N, K, T, seed=5)
    x64 = x.astype(np.float64)
    H = 2.0 * (x64.T @ x64) / T
    H[np.diag_indices(K)] += 0.01 * np.mean(np.diag(H))
    R = u @ H @ u.T
    assert np.abs(R - np.eye(K)).max() < 1e-8
    rows = np.random.default_rng(0).choice(N, 48, replace=False)
    _follow(wf, np.zeros(K, bool), u, q, rows=rows)
    s_ref = (np.abs(wf).max(axis=1) / np.float32(127)).astype(np.float32)
    assert np.array_equal(sch, s_ref)


def test_gptq_argument_checks():
    w = torch.zeros((8, 100), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((4, 100), dtype=torch.float32, device="cuda")
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED"):
        w8.w8a8_gptq_quantize(w, x)
    w = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(w8.W8A8Error, match="INVALID"):
        w8.w8a8_gptq_quantize(w, x, damp=0.0)
    # the codes are stored 16 bytes at a time: a misaligned wq is refused before any launch
    buf = torch.empty(8 * 128 + 16, dtype=torch.int8, device="cuda")
    with pytest.raises(w8.W8A8Error, match="ALIGNMENT"):
        w8.w8a8_gptq_quantize(w, x, wq=buf[1:1 + 8 * 128].view(8, 128))
