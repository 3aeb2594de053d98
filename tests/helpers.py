"""Shared test helpers: moving numpy inputs to the device and comparing against the oracle."""
import numpy as np
import torch

import oracle

SENTINEL_BF16 = 0x7FC1  # a NaN pattern no kernel writes
SENTINEL_I8 = -128       # a code the kernels never produce


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def with_canary(shape, dtype, fill):
    """An output tensor of `shape` carved from a larger buffer pre-filled with `fill`; the
    returned `check()` verifies every element beyond the tensor still holds `fill`'s bit
    pattern (compared as integers, so a NaN fill works too)."""
    n = int(np.prod(shape))
    buf = torch.full((n + 256,), fill, dtype=dtype, device="cuda")
    t = buf[:n].view(*shape)
    ibits = {1: torch.int8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[buf.element_size()]
    ref = buf[n:].clone().view(ibits)

    def check():
        assert torch.equal(buf[n:].view(ibits), ref), "write past the end of an output"
    return t, check


def bf16_out(shape):
    n = int(np.prod(shape))
    buf = torch.full((n + 256,), SENTINEL_BF16, dtype=torch.int16, device="cuda")
    t = buf[:n].view(torch.bfloat16).view(*shape)

    def check():
        assert bool((buf[n:] == SENTINEL_BF16).all()), "write past the end of an output"
    return t, check


def i8_out(shape):
    return with_canary(shape, torch.int8, SENTINEL_I8)


def f32_out(shape):
    return with_canary(shape, torch.float32, float("nan"))


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in representable bf16 steps between two bf16 bit-pattern arrays."""
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(ordered(a) - ordered(b))


def assert_rms_rows_match(got_q, got_s, x, gamma, eps, residual=None, ref=None,
                          ref_fn=oracle.smooth_rmsnorm_quant):
    """GPU smoothed-RMSNorm results against the oracle. Rows whose binary64 mean of squares
    lies so close to a binary32 rounding boundary that another summation order may round it
    the other way (oracle flag `ambiguous`) may match either neighbouring binary32 value;
    every other row must match exactly."""
    if ref is None:
        ref = ref_fn(x, gamma, eps, residual=residual)
    bad = np.where((got_s != ref["s"]) | (got_q != ref["q"]).any(axis=1))[0]
    for m in bad:
        assert ref["ambiguous"][m], f"row {m} differs and is not ambiguous"
        ok = False
        for direction in (np.inf, -np.inf):
            ms = ref["ms"].copy()
            ms[m] = np.nextafter(np.float32(ms[m]), np.float32(direction))
            alt = ref_fn(x[m:m + 1], gamma, eps,
                                              residual=None if residual is None
                                              else residual[m:m + 1],
                                              ms_override=ms[m:m + 1])
            if alt["s"][0] == got_s[m] and np.array_equal(alt["q"][0], got_q[m]):
                ok = True
        assert ok, f"row {m} matches neither admissible mean of squares"
    return ref, len(bad)


def check_block_rows(rows, x, attn, pr, eps, got):
    """One decoder block's chain on sampled rows, stage by stage: every stage's GPU result
    against the oracle applied to the GPU's own inputs of that stage, each of which the
    previous check has tied to the oracle. An order-ambiguous RMSNorm row, where the GPU may
    take the other admissible neighbouring mean of squares, is thus checked through the
    whole chain instead of being left out. `got` maps q1 s1 qkv q2 s2 o h q3 s3 q4 s4 down
    (and optionally gate_up, a) to host arrays (bf16 as uint16 bits, a as float32); returns
    how many RMSNorm rows took the other neighbour."""
    xr, ar = x[rows], attn[rows]
    g = {k: v[rows] for k, v in got.items()}

    def gemm(q, s, name):
        y, _ = oracle.gemm_dequant(q, s, pr[name]["wq"], pr[name]["s_ch"], want_acc=False)
        return y

    _, n1 = assert_rms_rows_match(g["q1"], g["s1"], xr, pr["gamma1f"], eps)
    assert np.array_equal(g["qkv"], gemm(g["q1"], g["s1"], "qkv"))
    q2, s2 = oracle.quantize_rows(ar, pr.get("s_inv_o"))
    assert np.array_equal(g["q2"], q2) and np.array_equal(g["s2"], s2)
    assert np.array_equal(g["o"], gemm(g["q2"], g["s2"], "o"))
    ref3, n3 = assert_rms_rows_match(g["q3"], g["s3"], g["o"], pr["gamma2f"], eps,
                                     residual=xr)
    assert np.array_equal(g["h"], ref3["h"])
    gu = gemm(g["q3"], g["s3"], "gate_up")
    if "gate_up" in g:
        assert np.array_equal(g["gate_up"], gu)
    if "a" in g:
        assert np.array_equal(g["a"].view(np.uint32), oracle.silu_mul(gu).view(np.uint32))
    q4, s4 = oracle.silu_mul_quant(gu)
    assert np.array_equal(g["q4"], q4) and np.array_equal(g["s4"], s4)
    assert np.array_equal(g["down"], gemm(g["q4"], g["s4"], "down"))
    return n1 + n3
