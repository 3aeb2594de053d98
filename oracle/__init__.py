"""Oracle for the W8A8 SmoothQuant linear path: TEST INFRASTRUCTURE ONLY.

A plain, slow CPU restatement (``oracle.c``) of what the path computes, with this thin
numpy/ctypes wrapper. Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import it; the library (``int8_w8a8_quantized_smoothed_b200``) never
does, and the two share no code. bf16 arrays are ``numpy.uint16`` bit patterns.

Parity pins (tests/test_oracle_pins.py) tie every function here to the pages' worked
examples, closed forms, invariants or brute force; see the header of ``oracle.c`` for the
passages each function follows.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None
NTHREADS = os.cpu_count() or 1


def lib():
    """Load (building first if needed) ``liboracle.so``."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        I64 = C.c_int64
        L.oracle_bf16_to_f32.restype = C.c_float
        L.oracle_bf16_to_f32.argtypes = [C.c_uint16]
        L.oracle_f32_to_bf16.restype = C.c_uint16
        L.oracle_f32_to_bf16.argtypes = [C.c_float]
        L.oracle_quantize_row_f32.argtypes = [P, I64, P, P]
        L.oracle_quantize_rows.argtypes = [P, P, I64, I64, P, P, C.c_int]
        L.oracle_e4m3_to_f32.restype = C.c_float
        L.oracle_e4m3_to_f32.argtypes = [C.c_uint8]
        L.oracle_f32_to_e4m3.restype = C.c_uint8
        L.oracle_f32_to_e4m3.argtypes = [C.c_float]
        L.oracle_quantize_row_f32_fp8.argtypes = [P, I64, P, P]
        L.oracle_quantize_rows_fp8.argtypes = [P, P, I64, I64, P, P, C.c_int]
        L.oracle_quantize_rows_f32_fp8.argtypes = [P, I64, I64, P, P, C.c_int]
        L.oracle_dequant_f32acc.argtypes = [P, P, P, I64, I64, P]
        L.oracle_gptq_hessian.argtypes = [P, I64, I64, C.c_double, P, P]
        L.oracle_gptq_hinv_chol.argtypes = [P, I64, P]
        L.oracle_gptq_quantize.argtypes = [P, I64, I64, P, P, P, P, P, P, C.c_double, P, C.c_int]
        L.oracle_gemm_fp8.argtypes = [P, P, P, P, I64, I64, I64, P, P, P, C.c_int]
        L.oracle_minmax_scale.restype = C.c_float
        L.oracle_minmax_scale.argtypes = [P, I64]
        L.oracle_quantize_rows_static.argtypes = [P, P, C.c_float, I64, I64, P, C.c_int]
        L.oracle_smooth_rmsnorm_quant.argtypes = [P, P, P, P, C.c_float, I64, I64, P, P, P, P,
                                                  P, P, C.c_int]
        L.oracle_exp.restype = C.c_float
        L.oracle_exp.argtypes = [C.c_float]
        L.oracle_silu.restype = C.c_float
        L.oracle_silu.argtypes = [C.c_float]
        L.oracle_silu_mul_quant.argtypes = [P, I64, I64, P, P, C.c_int]
        L.oracle_silu_mul.argtypes = [P, I64, I64, P, C.c_int]
        L.oracle_dequant.restype = C.c_uint16
        L.oracle_dequant.argtypes = [C.c_int32, C.c_float, C.c_float]
        L.oracle_gemm_dequant.argtypes = [P, P, P, P, I64, I64, I64, P, P, C.c_int]
        L.oracle_gemm_dequant_sampled.argtypes = [P, P, P, P, I64, P, P, I64, P, P]
        L.oracle_column_absmax_f32.argtypes = [P, I64, I64, P]
        L.oracle_column_absmax_bf16.argtypes = [P, I64, I64, P]
        L.oracle_smoothing_factors.argtypes = [P, P, I64, C.c_double, P]
        L.oracle_fold_gamma.argtypes = [P, P, I64, P, P]
        L.oracle_smooth_weight.argtypes = [P, P, I64, I64, P]
        L.oracle_rtn_weights.argtypes = [P, P, I64, I64, P, P, C.c_int]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


# ------------------------------------------------------------------ scalars


def bf16_to_f32(b):
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f):
    """Elementwise RN-even narrowing through the oracle's scalar routine."""
    f = np.asarray(f, dtype=np.float32)
    L = lib()
    out = np.empty(f.shape, dtype=np.uint16)
    flat_in, flat_out = f.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = L.oracle_f32_to_bf16(float(flat_in[i]))
    return out


def exp(x: float) -> float:
    return lib().oracle_exp(float(np.float32(x)))


def silu(g: float) -> float:
    return lib().oracle_silu(float(np.float32(g)))


def dequant(acc: int, s_tok: float, s_ch: float) -> int:
    return lib().oracle_dequant(int(acc), float(s_tok), float(s_ch))


# ------------------------------------------------------------------ row ops


def quantize_row_f32(y):
    """Per-token quantization of one fp32 row -> (q int8 [K], s float32)."""
    y = _c(y, np.float32)
    q = np.empty(y.shape[-1], dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    lib().oracle_quantize_row_f32(_p(y), y.shape[-1], _p(q), _p(s))
    return q, s[0]


def quantize_rows(x_bf16, sinv=None, nthreads=NTHREADS):
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    sinv = _c(sinv, np.float32)
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    lib().oracle_quantize_rows(_p(x), _p(sinv), M, K, _p(q), _p(s), nthreads)
    return q, s


def e4m3_to_f32(b: int) -> float:
    return lib().oracle_e4m3_to_f32(int(b))


def f32_to_e4m3(v: float) -> int:
    return int(lib().oracle_f32_to_e4m3(float(v)))


def quantize_row_f32_fp8(y):
    y = _c(y, np.float32)
    q = np.empty(y.shape[-1], dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    lib().oracle_quantize_row_f32_fp8(_p(y), y.shape[-1], _p(q), _p(s))
    return q, s[0]


def quantize_rows_fp8(x_bf16, sinv=None, nthreads=NTHREADS):
    """Per-token FP8 (E4M3) quantization -> (codes uint8 [M, K], scales float32 [M])."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    sinv = _c(sinv, np.float32)
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty(M, dtype=np.float32)
    lib().oracle_quantize_rows_fp8(_p(x), _p(sinv), M, K, _p(q), _p(s), nthreads)
    return q, s


def quantize_rows_f32_fp8(y, nthreads=NTHREADS):
    """Per-row FP8 quantization of fp32 rows -> (codes uint8 [M, K], scales float32 [M])."""
    y = _c(y, np.float32)
    M, K = y.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty(M, dtype=np.float32)
    lib().oracle_quantize_rows_f32_fp8(_p(y), M, K, _p(q), _p(s), nthreads)
    return q, s


def smooth_rmsnorm_quant_fp8(x_bf16, gamma, eps, residual=None, ms_override=None,
                             nthreads=NTHREADS):
    """The smoothed RMSNorm of ``smooth_rmsnorm_quant`` with FP8 per-token quantization."""
    r = smooth_rmsnorm_quant(x_bf16, gamma, eps, residual=residual, ms_override=ms_override,
                             want_y=True, quantize=False, nthreads=nthreads)
    r["q"], r["s"] = quantize_rows_f32_fp8(r["y"], nthreads)
    return r


def silu_mul_quant_fp8(gate_up_bf16, nthreads=NTHREADS):
    """silu(gate) * up with FP8 per-token quantization -> (codes, scales)."""
    return quantize_rows_f32_fp8(silu_mul(gate_up_bf16, nthreads), nthreads)


def rtn_weights_fp8(w_bf16, s=None, nthreads=NTHREADS):
    """FP8 round-to-nearest weights: rows (output channels) of W * diag(s) quantized to E4M3
    with per-channel scales absmax / 448 -> (codes uint8 [N, K], s_ch float32 [N])."""
    w = _c(w_bf16, np.uint16)
    v = smooth_weight(w, s) if s is not None else bf16_to_f32(w)
    return quantize_rows_f32_fp8(v, nthreads)


def dequant_f32acc(acc, s_tok, s_ch):
    """bf16 bits of (acc * s_tok[m]) * s_ch[n] for binary32 accumulators acc [M, N]."""
    acc = _c(acc, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.uint16)
    lib().oracle_dequant_f32acc(_p(acc), _p(_c(s_tok, np.float32)), _p(_c(s_ch, np.float32)),
                                M, N, _p(y))
    return y


def gemm_fp8(xq, s_tok, wq, s_ch, nthreads=NTHREADS):
    """FP8 GEMM reference -> (y bf16 bits [M, N], exact acc float64, sum |products| float64)."""
    xq = _c(xq, np.uint8)
    wq = _c(wq, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    st = _c(s_tok, np.float32)
    sc = _c(s_ch, np.float32)
    acc = np.empty((M, N), dtype=np.float64)
    absacc = np.empty((M, N), dtype=np.float64)
    y = np.empty((M, N), dtype=np.uint16)
    lib().oracle_gemm_fp8(_p(xq), _p(st), _p(wq), _p(sc), M, N, K, _p(acc), _p(absacc), _p(y),
                          nthreads)
    return y, acc, absacc


def minmax_scale(values_f32):
    """Symmetric min-max calibration scale S = max(|min|, |max|) / 127 of a tensor."""
    v = _c(values_f32, np.float32).ravel()
    return np.float32(lib().oracle_minmax_scale(_p(v), v.size))


def quantize_rows_static(x_bf16, scale, sinv=None, nthreads=NTHREADS):
    """Static per-tensor quantization with a fixed scale -> q int8 [M, K]."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    sinv = _c(sinv, np.float32)
    q = np.empty((M, K), dtype=np.int8)
    rc = lib().oracle_quantize_rows_static(_p(x), _p(sinv), float(scale), M, K, _p(q), nthreads)
    if rc != 0:
        raise ValueError("scale must be > 0")
    return q


def smooth_rmsnorm_quant(x_bf16, gamma, eps, residual=None, ms_override=None,
                         want_y=False, quantize=True, nthreads=NTHREADS):
    """Returns dict(q, s, h (bf16 or None), ms, ambiguous, y (fp32 or None))."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    r = _c(residual, np.uint16)
    g = _c(gamma, np.float32)
    h = np.empty((M, K), dtype=np.uint16) if r is not None else None
    q = np.empty((M, K), dtype=np.int8) if quantize else None
    s = np.empty(M, dtype=np.float32) if quantize else None
    ms = np.empty(M, dtype=np.float32)
    amb = np.zeros(M, dtype=np.uint8)
    mo = _c(ms_override, np.float32)
    y = np.empty((M, K), dtype=np.float32) if want_y else None
    lib().oracle_smooth_rmsnorm_quant(_p(x), _p(r), _p(h), _p(g), float(eps), M, K, _p(q),
                                      _p(s), _p(ms), _p(amb), _p(mo), _p(y), nthreads)
    return dict(q=q, s=s, h=h, ms=ms, ambiguous=amb.astype(bool), y=y)


def silu_mul(gate_up_bf16, nthreads=NTHREADS):
    """a = silu(gate) * up (binary32 [M, I]) of a [M, 2I] gate|up bf16 tensor."""
    gu = _c(gate_up_bf16, np.uint16)
    M, I2 = gu.shape
    a = np.empty((M, I2 // 2), dtype=np.float32)
    lib().oracle_silu_mul(_p(gu), M, I2 // 2, _p(a), nthreads)
    return a


def silu_mul_quant(gate_up_bf16, nthreads=NTHREADS):
    gu = _c(gate_up_bf16, np.uint16)
    M, I2 = gu.shape
    assert I2 % 2 == 0
    I = I2 // 2
    q = np.empty((M, I), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    lib().oracle_silu_mul_quant(_p(gu), M, I, _p(q), _p(s), nthreads)
    return q, s


# ------------------------------------------------------------------ GEMM


def gemm_dequant(xq, s_tok, wq, s_ch, want_acc=True, nthreads=NTHREADS):
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    st = _c(s_tok, np.float32)
    sc = _c(s_ch, np.float32)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    y = np.empty((M, N), dtype=np.uint16)
    acc = np.empty((M, N), dtype=np.int32) if want_acc else None
    lib().oracle_gemm_dequant(_p(xq), _p(st), _p(wq), _p(sc), M, N, K, _p(y), _p(acc),
                              nthreads)
    return y, acc


def gemm_dequant_sampled(xq, s_tok, wq, s_ch, ms, ns):
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    st = _c(s_tok, np.float32)
    sc = _c(s_ch, np.float32)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    K = xq.shape[1]
    y = np.empty(ms.size, dtype=np.uint16)
    acc = np.empty(ms.size, dtype=np.int32)
    lib().oracle_gemm_dequant_sampled(_p(xq), _p(st), _p(wq), _p(sc), K, _p(ms), _p(ns),
                                      ms.size, _p(y), _p(acc))
    return y, acc


# ------------------------------------------------------------------ offline prep


def column_absmax_f32(a):
    a = _c(a, np.float32)
    M, K = a.shape
    out = np.empty(K, dtype=np.float32)
    lib().oracle_column_absmax_f32(_p(a), M, K, _p(out))
    return out


def column_absmax_bf16(b):
    b = _c(b, np.uint16)
    M, K = b.shape
    out = np.empty(K, dtype=np.float32)
    lib().oracle_column_absmax_bf16(_p(b), M, K, _p(out))
    return out


def smoothing_factors(a_max, w_max, alpha):
    a = _c(a_max, np.float32)
    w = _c(w_max, np.float32)
    s = np.empty(a.size, dtype=np.float32)
    lib().oracle_smoothing_factors(_p(a), _p(w), a.size, float(alpha), _p(s))
    return s


def fold_gamma(gamma, s):
    g = _c(gamma, np.float32)
    s = _c(s, np.float32)
    gf = np.empty(g.size, dtype=np.float32)
    si = np.empty(g.size, dtype=np.float32)
    lib().oracle_fold_gamma(_p(g), _p(s), g.size, _p(gf), _p(si))
    return gf, si


def smooth_weight(w_bf16, s):
    w = _c(w_bf16, np.uint16)
    N, K = w.shape
    s = _c(s, np.float32)
    out = np.empty((N, K), dtype=np.float32)
    lib().oracle_smooth_weight(_p(w), _p(s), N, K, _p(out))
    return out


def rtn_weights(w_bf16, s=None, nthreads=NTHREADS):
    w = _c(w_bf16, np.uint16)
    N, K = w.shape
    s = _c(s, np.float32)
    wq = np.empty((N, K), dtype=np.int8)
    s_ch = np.empty(N, dtype=np.float32)
    lib().oracle_rtn_weights(_p(w), _p(s), N, K, _p(wq), _p(s_ch), nthreads)
    return wq, s_ch


# ------------------------------------------------------------------ composite prep


def prepare_linear(x_cal_f32, w_bf16, alpha, nthreads=NTHREADS):
    """SmoothQuant + per-channel RTN for one linear whose input activations are x_cal:
    returns dict(s, s_inv, wq, s_ch). The weight W [N, K] is scaled by s on its input
    channels before RTN."""
    a_max = column_absmax_f32(x_cal_f32)
    w_max = column_absmax_bf16(w_bf16)
    s = smoothing_factors(a_max, w_max, alpha)
    _, s_inv = fold_gamma(np.ones_like(s), s)
    wq, s_ch = rtn_weights(w_bf16, s, nthreads)
    return dict(s=s, s_inv=s_inv, wq=wq, s_ch=s_ch)


def block_reference(inputs, prep, eps, nthreads=NTHREADS):
    """One decoder block's linear path (the chain of the M=512 block workload) on the CPU.

    inputs: dict(x bf16 [M,H], attn bf16 [M,H]); prep: dict with per-linear wq/s_ch and
    gamma1f/gamma2f (folded gammas) and s_inv_o (or None). Returns every intermediate."""
    out = {}
    r1 = smooth_rmsnorm_quant(inputs["x"], prep["gamma1f"], eps, nthreads=nthreads)
    out["q1"], out["s1"], out["amb1"] = r1["q"], r1["s"], r1["ambiguous"]
    out["qkv"], _ = gemm_dequant(r1["q"], r1["s"], prep["qkv"]["wq"], prep["qkv"]["s_ch"],
                                 want_acc=False, nthreads=nthreads)
    out["q2"], out["s2"] = quantize_rows(inputs["attn"], prep.get("s_inv_o"),
                                         nthreads=nthreads)
    out["o"], _ = gemm_dequant(out["q2"], out["s2"], prep["o"]["wq"], prep["o"]["s_ch"],
                               want_acc=False, nthreads=nthreads)
    r2 = smooth_rmsnorm_quant(out["o"], prep["gamma2f"], eps, residual=inputs["x"],
                              nthreads=nthreads)
    out["h"], out["q3"], out["s3"], out["amb3"] = r2["h"], r2["q"], r2["s"], r2["ambiguous"]
    out["gate_up"], _ = gemm_dequant(r2["q"], r2["s"], prep["gate_up"]["wq"],
                                     prep["gate_up"]["s_ch"], want_acc=False,
                                     nthreads=nthreads)
    out["q4"], out["s4"] = silu_mul_quant(out["gate_up"], nthreads=nthreads)
    out["down"], _ = gemm_dequant(out["q4"], out["s4"], prep["down"]["wq"],
                                  prep["down"]["s_ch"], want_acc=False, nthreads=nthreads)
    return out


# ------------------------------------------------------------------ GPTQ


def gptq_hessian(x_f32, damp=0.01):
    """H = (2/T) X^T X with dead columns set to 1 and dampening -> (H float64 [K, K], dead)."""
    x = _c(x_f32, np.float32)
    T, K = x.shape
    H = np.empty((K, K), dtype=np.float64)
    dead = np.empty(K, dtype=np.uint8)
    lib().oracle_gptq_hessian(_p(x), T, K, float(damp), _p(H), _p(dead))
    return H, dead.astype(bool)


def gptq_hinv_chol(H):
    """U upper triangular with H^-1 = U^T U."""
    H = _c(H, np.float64)
    K = H.shape[0]
    U = np.empty((K, K), dtype=np.float64)
    if lib().oracle_gptq_hinv_chol(_p(H), K, _p(U)) != 0:
        raise ValueError("H is not positive definite")
    return U


def gptq_quantize(w_f32, dead, U, q_follow=None, tie_tol=0.0, want_wcomp=False,
                  nthreads=NTHREADS):
    """Column-by-column GPTQ of the rows of w [N, K] -> dict(q, s, wcomp, status)."""
    w = _c(w_f32, np.float32)
    N, K = w.shape
    d = _c(np.asarray(dead, dtype=np.uint8), np.uint8)
    U = _c(U, np.float64)
    q = np.empty((N, K), dtype=np.int8)
    s = np.empty(N, dtype=np.float32)
    wc = np.empty((N, K), dtype=np.float64) if want_wcomp else None
    qf = _c(q_follow, np.int8)
    st = np.empty((N, K), dtype=np.uint8) if q_follow is not None else None
    lib().oracle_gptq_quantize(_p(w), N, K, _p(d), _p(U), _p(q), _p(s), _p(wc), _p(qf),
                               float(tie_tol), _p(st), nthreads)
    return dict(q=q, s=s, wcomp=wc, status=st)


def gptq(w_f32, x_f32, damp=0.01, want_wcomp=False, nthreads=NTHREADS):
    """GPTQ int8 weights of w [N, K] (binary32, smoothed) for calibration inputs x [T, K]."""
    H, dead = gptq_hessian(x_f32, damp)
    U = gptq_hinv_chol(H)
    r = gptq_quantize(w_f32, dead, U, want_wcomp=want_wcomp, nthreads=nthreads)
    r.update(H=H, dead=dead, U=U)
    return r
