"""Parity of the fused decoder-block kernel (w8a8_block_decode: the whole linear path of a
Llama-3.1-8B block at decode sizes in one persistent launch) with the oracle, and with the
chain of separate kernels it replaces. Every intermediate is compared bit-exactly on sampled
rows (rows are independent), stage by stage against the oracle applied to the kernel's own
inputs of that stage; a row whose RMSNorm mean of squares is order-ambiguous (oracle flag)
may take either admissible neighbour and is then checked through the rest of the chain."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import prep, synth
from helpers import check_block_rows, dev, dev_bf16, host, host_bf16
from test_gpu_block import EPS, _block_prep

pytestmark = pytest.mark.gpu

H, I = 4096, 14336


@pytest.fixture(scope="module")
def block():
    pr = _block_prep(H, I, seed=300)
    d = {k: (dev(v["wq"]), dev(v["s_ch"])) for k, v in pr.items() if isinstance(v, dict)}
    d["gate_up_il"] = prep.interleave_gate_up(*d["gate_up"])
    return pr, d


def _fused(d, pr, x, attn, buffers=None):
    return w8.w8a8_block_decode(dev_bf16(x), dev_bf16(attn), dev(pr["gamma1f"]),
                                dev(pr["s_inv_o"]), dev(pr["gamma2f"]), d["qkv"], d["o"],
                                d["gate_up_il"], d["down"], EPS, buffers=buffers)


@pytest.mark.parametrize("M", [1, 8, 16, 33, 64])
def test_fused_block_matches_oracle(block, M):
    pr, d = block
    x = synth.activation(M, H, 400 + M)
    attn = synth.activation(M, H, 500 + M)
    b = _fused(d, pr, x, attn)
    torch.cuda.synchronize()
    assert w8.w8a8_device_status() == 0
    rows = np.unique(np.concatenate([[0, M - 1], synth.row_sample(M, M, count=4)]))
    got = dict(q1=host(b.q[0]), s1=host(b.s[0]), qkv=host_bf16(b.qkv), q2=host(b.q[1]),
               s2=host(b.s[1]), o=host_bf16(b.o), h=host_bf16(b.h), q3=host(b.q[2]),
               s3=host(b.s[2]), a=host(b.a), q4=host(b.q[3]), s4=host(b.s[3]),
               down=host_bf16(b.y))
    check_block_rows(rows, x, attn, pr, EPS, got)
    ref = oracle.block_reference({"x": x[rows], "attn": attn[rows]}, pr, EPS)
    keep = ~(ref["amb1"] | ref["amb3"])
    r = rows[keep]
    assert np.array_equal(host(b.q[0])[r], ref["q1"][keep])
    assert np.array_equal(host(b.s[0])[r], ref["s1"][keep])
    assert np.array_equal(host_bf16(b.qkv)[r], ref["qkv"][keep])
    assert np.array_equal(host(b.q[1])[rows], ref["q2"])
    assert np.array_equal(host(b.s[1])[rows], ref["s2"])
    assert np.array_equal(host_bf16(b.o)[rows], ref["o"])
    assert np.array_equal(host_bf16(b.h)[rows], ref["h"])
    assert np.array_equal(host(b.q[2])[r], ref["q3"][keep])
    assert np.array_equal(host(b.s[2])[r], ref["s3"][keep])
    a_ref = oracle.silu_mul(ref["gate_up"])
    assert np.array_equal(host(b.a)[r].view(np.uint32), a_ref[keep].view(np.uint32))
    assert np.array_equal(host(b.q[3])[r], ref["q4"][keep])
    assert np.array_equal(host(b.s[3])[r], ref["s4"][keep])
    assert np.array_equal(host_bf16(b.y)[r], ref["down"][keep])


def test_fused_block_equals_separate_kernels_and_repeats(block):
    pr, d = block
    M = 40
    x = synth.activation(M, H, 77)
    attn = synth.activation(M, H, 78)
    xd, ad = dev_bf16(x), dev_bf16(attn)
    q1, s1 = w8.w8a8_smooth_rmsnorm_quant(xd, dev(pr["gamma1f"]), EPS)
    qkv = w8.w8a8_gemm_dequant(q1, s1, *d["qkv"])
    q2, s2 = w8.w8a8_quantize_rows(ad, dev(pr["s_inv_o"]))
    o = w8.w8a8_gemm_dequant(q2, s2, *d["o"])
    q3, s3, h = w8.w8a8_smooth_rmsnorm_quant(o, dev(pr["gamma2f"]), EPS, residual=xd)
    q4, s4, a = w8.w8a8_gemm_silu_quant(q3, s3, *d["gate_up_il"])
    y = w8.w8a8_gemm_dequant(q4, s4, *d["down"])
    bufs = w8.BlockBuffers(M, H, I, 6144, xd.device)
    for _ in range(3):  # the workspace comes back ready for the next call
        b = _fused(d, pr, x, attn, buffers=bufs)
        torch.cuda.synchronize()
        assert w8.w8a8_device_status() == 0
        # the RMSNorm sums may round differently only on order-ambiguous rows (none expected)
        assert torch.equal(b.s[0], s1) and torch.equal(b.q[0], q1)
        assert torch.equal(b.qkv, qkv) and torch.equal(b.o, o) and torch.equal(b.h, h)
        assert torch.equal(b.q[2], q3) and torch.equal(b.s[2], s3)
        assert torch.equal(b.a.view(torch.int32), a.view(torch.int32))
        assert torch.equal(b.q[3], q4) and torch.equal(b.s[3], s4)
        assert torch.equal(b.y, y)


def test_fused_block_in_a_cuda_graph(block):
    pr, d = block
    M = 8
    x = synth.activation(M, H, 91)
    attn = synth.activation(M, H, 92)
    bufs = w8.BlockBuffers(M, H, I, 6144, torch.device("cuda"))
    xd, ad = dev_bf16(x), dev_bf16(attn)
    args = (xd, ad, dev(pr["gamma1f"]), dev(pr["s_inv_o"]), dev(pr["gamma2f"]), d["qkv"], d["o"],
            d["gate_up_il"], d["down"], EPS)
    w8.w8a8_block_decode(*args, buffers=bufs)
    torch.cuda.synchronize()
    y0 = bufs.y.clone()
    bufs.y.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            w8.w8a8_block_decode(*args, buffers=bufs, stream=s)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    assert w8.w8a8_device_status() == 0
    assert torch.equal(bufs.y, y0)


def test_fused_block_argument_checks(block):
    pr, d = block
    x = synth.activation(65, H, 1)
    with pytest.raises(w8.W8A8Error, match="UNSUPPORTED"):
        _fused(d, pr, x, x)
