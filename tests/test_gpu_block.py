"""End-to-end parity on the workloads: the single smoothed linear (M=16, K=256, N=512, 4 outlier
channels) and one Llama-3.1-8B decoder block's linear path at M=512 (smoothed RMSNorm+quant ->
qkv; attention stand-in -> quant -> o; residual add -> smoothed RMSNorm+quant -> gate_up ->
SiLU*up+quant -> down). Every intermediate is compared bit-exactly with the oracle; the block
is checked on a seeded sample of rows (all ops are per token, so rows are independent)."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import prep, synth
from helpers import assert_rms_rows_match, check_block_rows, dev, dev_bf16, host, host_bf16

pytestmark = pytest.mark.gpu

EPS = 1e-5
ALPHA = 0.5


def test_single_smoothed_linear():
    M, K, N = 16, 256, 512
    x = synth.activation(M, K, 0, outliers=4)
    w = synth.weight(N, K, 1)
    p = oracle.prepare_linear(oracle.bf16_to_f32(x), w, ALPHA)  # calibrate on X itself
    q_ref, s_ref = oracle.quantize_rows(x, p["s_inv"])
    y_ref, acc_ref = oracle.gemm_dequant(q_ref, s_ref, p["wq"], p["s_ch"])

    q, s = w8.w8a8_quantize_rows(dev_bf16(x), dev(p["s_inv"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = w8.w8a8_gemm_dequant(q, s, dev(p["wq"]), dev(p["s_ch"]), acc_out=acc)
    assert np.array_equal(host(q), q_ref) and np.array_equal(host(s), s_ref)
    assert np.array_equal(host(acc), acc_ref)
    assert np.array_equal(host_bf16(y), y_ref)

    # the W8A8 output approximates the bf16 layer; smoothing makes it markedly better
    ref = oracle.bf16_to_f32(x).astype(np.float64) @ oracle.bf16_to_f32(w).astype(np.float64).T
    err_s = np.linalg.norm(oracle.bf16_to_f32(y_ref) - ref) / np.linalg.norm(ref)
    q0, s0 = oracle.quantize_rows(x)
    wq0, sc0 = oracle.rtn_weights(w)
    y0, _ = oracle.gemm_dequant(q0, s0, wq0, sc0)
    err_0 = np.linalg.norm(oracle.bf16_to_f32(y0) - ref) / np.linalg.norm(ref)
    assert err_s < 0.05 and err_s < err_0


def test_product_prep_matches_oracle_prep():
    K, N = 4096, 1024
    xc = synth.activation(128, K, 3)
    w = synth.weight(N, K, 4)
    gam = synth.gamma(K, 5)
    p = oracle.prepare_linear(oracle.bf16_to_f32(xc), w, ALPHA)
    d = prep.prepare_linear(dev_bf16(w), prep.column_absmax(dev_bf16(xc)), ALPHA)
    assert np.array_equal(d["s"], p["s"])
    assert np.array_equal(d["s_inv"], p["s_inv"])
    assert np.array_equal(host(d["wq"]), p["wq"]) and np.array_equal(host(d["s_ch"]), p["s_ch"])
    gf_o, _ = oracle.fold_gamma(gam, p["s"])
    gf_p, _ = prep.fold(gam, d["s"])
    assert np.array_equal(gf_o, gf_p)


def _block_prep(H, I, seed, C=128):
    """Oracle-side prep of one decoder block: calibration batches of C tokens."""
    ws = {n: synth.weight(N, K, seed + i) for i, (n, N, K) in enumerate(
        [("qkv", 6144, H), ("o", H, H), ("gate_up", 2 * I, H), ("down", H, I)])}
    g1 = synth.gamma(H, seed + 10)
    g2 = synth.gamma(H, seed + 11)
    xc = synth.activation(C, H, seed + 20)
    ac = synth.activation(C, H, seed + 21)
    hc = synth.activation(C, H, seed + 22)
    a1 = oracle.smooth_rmsnorm_quant(xc, g1, EPS, want_y=True, quantize=False)["y"]
    a3 = oracle.smooth_rmsnorm_quant(hc, g2, EPS, want_y=True, quantize=False)["y"]
    out = {}
    p = oracle.prepare_linear(a1, ws["qkv"], ALPHA)
    out["qkv"] = p
    out["gamma1f"], _ = oracle.fold_gamma(g1, p["s"])
    out["o"] = oracle.prepare_linear(oracle.bf16_to_f32(ac), ws["o"], ALPHA)
    out["s_inv_o"] = out["o"]["s_inv"]
    p = oracle.prepare_linear(a3, ws["gate_up"], ALPHA)
    out["gate_up"] = p
    out["gamma2f"], _ = oracle.fold_gamma(g2, p["s"])
    wq, sch = oracle.rtn_weights(ws["down"])  # SiLU output: no norm to fold into
    out["down"] = dict(wq=wq, s_ch=sch)
    return out


def test_decoder_block_chain_m512_sampled_rows():
    H, I, M = 4096, 14336, 512
    pr = _block_prep(H, I, seed=100)
    x = synth.activation(M, H, 200)
    attn = synth.activation(M, H, 201)
    rows = synth.row_sample(M, 7, count=14)

    # GPU: the whole batch through the C ABI, one stream, no host sync inside
    d = {k: (dev(v["wq"]), dev(v["s_ch"])) for k, v in pr.items()
         if isinstance(v, dict)}
    xd, ad = dev_bf16(x), dev_bf16(attn)
    q1, s1 = w8.w8a8_smooth_rmsnorm_quant(xd, dev(pr["gamma1f"]), EPS)
    qkv = w8.w8a8_gemm_dequant(q1, s1, *d["qkv"])
    q2, s2 = w8.w8a8_quantize_rows(ad, dev(pr["s_inv_o"]))
    o = w8.w8a8_gemm_dequant(q2, s2, *d["o"])
    q3, s3, h = w8.w8a8_smooth_rmsnorm_quant(o, dev(pr["gamma2f"]), EPS, residual=xd)
    gu = w8.w8a8_gemm_dequant(q3, s3, *d["gate_up"])
    q4, s4 = w8.w8a8_silu_mul_quant(gu)
    down = w8.w8a8_gemm_dequant(q4, s4, *d["down"])
    torch.cuda.synchronize()
    assert w8.w8a8_device_status() == 0

    # every sampled row, stage by stage (ambiguous RMSNorm rows by the neighbour rule)
    got = dict(q1=host(q1), s1=host(s1), qkv=host_bf16(qkv), q2=host(q2), s2=host(s2),
               o=host_bf16(o), h=host_bf16(h), q3=host(q3), s3=host(s3),
               gate_up=host_bf16(gu), q4=host(q4), s4=host(s4), down=host_bf16(down))
    check_block_rows(rows, x, attn, pr, EPS, got)
    # and end to end from the inputs through the oracle's own chain
    ref = oracle.block_reference({"x": x[rows], "attn": attn[rows]}, pr, EPS)
    ambiguous = ref["amb1"] | ref["amb3"]
    assert ambiguous.sum() <= 1
    keep = ~ambiguous
    r = rows[keep]
    assert np.array_equal(host(q1)[r], ref["q1"][keep])
    assert np.array_equal(host(s1)[r], ref["s1"][keep])
    assert np.array_equal(host_bf16(qkv)[r], ref["qkv"][keep])
    assert np.array_equal(host(q2)[rows], ref["q2"]) and np.array_equal(host(s2)[rows], ref["s2"])
    assert np.array_equal(host_bf16(o)[rows], ref["o"])
    assert np.array_equal(host_bf16(h)[rows], ref["h"])
    assert np.array_equal(host(q3)[r], ref["q3"][keep])
    assert np.array_equal(host(s3)[r], ref["s3"][keep])
    assert np.array_equal(host_bf16(gu)[r], ref["gate_up"][keep])
    assert np.array_equal(host(q4)[r], ref["q4"][keep])
    assert np.array_equal(host(s4)[r], ref["s4"][keep])
    assert np.array_equal(host_bf16(down)[r], ref["down"][keep])
