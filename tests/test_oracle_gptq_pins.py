"""Pins for the oracle's GPTQ weight quantization (CPU only).

The pages describe GPTQ in prose (W8A8 "The solution: How GPTQ improves on naive
quantization"; a dampening factor in the AutoGPTQ article's "Crucial Config Tips"); the
oracle follows the GPTQ paper's arithmetic. These pins tie it to what the mathematics fixes:
the inverse-Hessian factor against LAPACK, the reduction to round-to-nearest when the
Hessian is diagonal, the compensated weights against the closed-form optimal-brain-surgeon
update solved directly, the layer-output error against RTN's, and the follow mode's verdicts.
"""
import numpy as np
import pytest

import oracle
from int8_w8a8_quantized_smoothed_b200 import synth


def _correlated(T, K, seed, rho=0.6):
    """Calibration activations with correlated channels and a few outlier channels."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, K))
    mix = np.eye(K) + rho * rng.standard_normal((K, K)) / np.sqrt(K)
    x = z @ mix
    x[:, rng.choice(K, max(1, K // 50), replace=False)] *= 20.0
    return x.astype(np.float32)


def _weights(N, K, seed):
    return (np.random.default_rng(seed).standard_normal((N, K)) * 0.02).astype(np.float32)


def test_hessian_closed_forms():
    # one token: H = 2 x x^T (rank one) plus the dampening on the diagonal
    x = np.array([[1.0, -2.0, 0.5, 0.0]], np.float32)
    H, dead = oracle.gptq_hessian(x, damp=0.0)
    assert list(dead) == [False, False, False, True]
    want = 2.0 * np.outer(x[0], x[0])
    want[3, 3] = 1.0  # dead channel
    assert np.array_equal(H, want)
    # orthogonal columns of norms c_j: H = diag(2 c_j^2 / T), then + damp * mean
    T = 8
    x = np.zeros((T, 3), np.float32)
    x[0, 0], x[1, 1], x[2, 2], x[3, 2] = 3.0, 1.0, 2.0, 2.0
    H, _ = oracle.gptq_hessian(x, damp=0.1)
    d = np.array([2 * 9 / T, 2 * 1 / T, 2 * 8 / T])
    assert np.allclose(H, np.diag(d + 0.1 * d.mean()), rtol=0, atol=1e-15)


@pytest.mark.parametrize("K", [7, 64, 200])
def test_inverse_hessian_factor_matches_lapack(K):
    H, _ = oracle.gptq_hessian(_correlated(4 * K, K, K), damp=0.01)
    U = oracle.gptq_hinv_chol(H)
    ref = np.linalg.cholesky(np.linalg.inv(H)).T  # upper, H^-1 = ref^T ref
    assert np.allclose(U, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    assert np.array_equal(U, np.triu(U)) and (np.diag(U) > 0).all()


def test_diagonal_hessian_reduces_to_rtn():
    """Orthogonal input channels: U is diagonal, no error reaches another column, so GPTQ is
    exactly per-channel round-to-nearest (itself pinned to the pages' worked examples)."""
    K, N = 32, 24
    q_mat, _ = np.linalg.qr(np.random.default_rng(1).standard_normal((64, K)))
    x = (q_mat * np.linspace(0.5, 4.0, K)).astype(np.float32)
    H, _ = oracle.gptq_hessian(x, 0.01)
    off = H - np.diag(np.diag(H))
    assert np.abs(off).max() < 1e-6 * np.abs(H).max()
    # make it exactly diagonal (the rounding of the float32 inputs leaves ~1e-8 residue)
    U = np.diag(1.0 / np.sqrt(np.diag(H)))
    w_bf16 = synth.weight(N, K, 3)
    w = oracle.bf16_to_f32(w_bf16)
    r = oracle.gptq_quantize(w, np.zeros(K, bool), U)
    q_rtn, s_rtn = oracle.rtn_weights(w_bf16)
    assert np.array_equal(r["q"], q_rtn) and np.array_equal(r["s"], s_rtn)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_compensation_is_the_closed_form_obs_update(seed):
    """When column j is quantized, the remaining weights F = {j..K-1} hold the minimizer of
    the layer-output error given the quantized columns P = {0..j-1}:
        w_F' = w_F + H_FF^-1 H_FP (w_P - q_P s)
    solved here directly with LAPACK, for every j."""
    K, N = 12, 5
    x = _correlated(48, K, seed)
    w = _weights(N, K, seed + 10)
    r = oracle.gptq(w, x, damp=0.01, want_wcomp=True)
    H, q, s = r["H"], r["q"].astype(np.float64), r["s"].astype(np.float64)
    for n in range(N):
        for j in range(1, K):
            P, F = np.arange(j), np.arange(j, K)
            dP = w[n, P].astype(np.float64) - q[n, P] * s[n]
            wF = w[n, F] + np.linalg.solve(H[np.ix_(F, F)], H[np.ix_(F, P)] @ dP)
            assert abs(r["wcomp"][n, j] - wF[0]) <= 1e-9 * max(1.0, abs(wF[0])), (n, j)


def test_gptq_output_error_below_rtn():
    K, N, T = 128, 64, 512
    x = _correlated(T, K, 5)
    w = _weights(N, K, 6)
    r = oracle.gptq(w, x, damp=0.01)
    wb = w.astype(np.float64)
    x64 = x.astype(np.float64)

    def err(q, s):
        return np.sum(((wb - q * s[:, None]) @ x64.T) ** 2)

    s_rtn = (np.abs(w).max(axis=1) / np.float32(127)).astype(np.float32)
    q_rtn = np.clip(np.rint(wb / s_rtn[:, None]), -127, 127)
    assert np.array_equal(r["s"], s_rtn)
    e_g, e_r = err(r["q"], r["s"].astype(np.float64)), err(q_rtn, s_rtn.astype(np.float64))
    assert e_g < 0.9 * e_r, (e_g, e_r)  # 0.80 of RTN on this draw
    assert np.abs(r["q"].astype(int)).max() <= 127


def test_follow_mode_verdicts_and_dead_channels():
    K, N = 48, 6
    x = _correlated(96, K, 7)
    x[:, 5] = 0.0  # a dead input channel
    w = _weights(N, K, 8)
    r = oracle.gptq(w, x)
    assert r["dead"][5] and not r["dead"][:5].any()
    assert (r["q"][:, 5] == 0).all() and np.isfinite(r["U"]).all()
    f = oracle.gptq_quantize(w, r["dead"], r["U"], q_follow=r["q"], tie_tol=1e-9)
    assert np.array_equal(f["q"], r["q"]) and not f["status"].any()
    bad = r["q"].copy()
    bad[2, 10] = np.clip(bad[2, 10] + 2, -127, 127) if bad[2, 10] < 120 else bad[2, 10] - 2
    f = oracle.gptq_quantize(w, r["dead"], r["U"], q_follow=bad, tie_tol=1e-9)
    assert f["status"][2, 10] == 2 and not f["status"][:2].any()
    assert not f["status"][2, :10].any()
