"""B200 (sm_100a) W8A8 SmoothQuant linear path: thin Python binding of ``libw8a8.so``.

The functions below carry the C ABI's names (``include/w8a8.h``) and only marshal
arguments: they check dtypes, shapes, devices and contiguity of torch tensors, pass raw
device pointers and the current CUDA stream, and raise ``W8A8Error`` on a non-zero status.
Every computation runs in the library's CUDA kernels; there is no CPU path. Importing the
package does not need a GPU, but every compute call does.

    q, s = w8a8_smooth_rmsnorm_quant(x, gamma_smoothed, eps)
    y = w8a8_gemm_dequant(q, s, wq, s_ch)
"""
import ctypes as C
import os
import threading

import torch

__all__ = [
    "W8A8Error", "lib", "LIB_PATH",
    "w8a8_quantize_rows", "w8a8_quantize_rows_static", "w8a8_smooth_rmsnorm_quant", "w8a8_silu_mul_quant",
    "w8a8_gemm_dequant", "w8a8_gemm_dequant_ex", "w8a8_gemm_workspace_size",
    "w8a8_gemm_workspace_size_ex", "w8a8_gemm_dequant_noalloc", "w8a8_gemm_silu_quant",
    "w8a8_gemm_silu_quant_workspace_size", "w8a8_gemm_rmsnorm_quant",
    "w8a8_gemm_rmsnorm_quant_workspace_size", "w8a8_gemm_rmsnorm_quant_one_launch_ok",
    "w8a8_probe_i8_mma", "w8a8_selftest_wait_timeout", "w8a8_set_overlap",
    "w8a8_get_overlap", "w8a8_device_status", "w8a8_last_device_status",
    "w8a8_status_string", "w8a8_version",
    "w8a8_quantize_rows_fp8", "w8a8_smooth_rmsnorm_quant_fp8", "w8a8_silu_mul_quant_fp8",
    "w8a8_gemm_dequant_fp8", "w8a8_gemm_fp8_workspace_size", "w8a8_gemm_silu_quant_fp8",
    "w8a8_gemm_silu_quant_fp8_workspace_size",
    "w8a8_gptq_quantize", "w8a8_gptq_workspace_size", "w8a8_probe_f64_fma",
    "w8a8_block_decode", "w8a8_block_decode_workspace_size", "BlockBuffers",
    "Workspace", "FP8",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw8a8.so")

STATUS = {0: "W8A8_OK", -1: "W8A8_ERR_INVALID_ARG", -2: "W8A8_ERR_ALIGNMENT",
          -3: "W8A8_ERR_UNSUPPORTED_SHAPE", -4: "W8A8_ERR_WORKSPACE", -5: "W8A8_ERR_CUDA",
          -6: "W8A8_ERR_TIMEOUT", -7: "W8A8_ERR_NO_DEVICE", -8: "W8A8_ERR_NUMERIC"}

# (name, restype, argtypes) of every function declared in include/w8a8.h
_P, _I64, _I, _F, _SZ = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
SIGNATURES = [
    ("w8a8_quantize_rows", _I, [_P, _P, _I64, _I64, _P, _P, _P]),
    ("w8a8_quantize_rows_static", _I, [_P, _P, _F, _I64, _I64, _P, _P, _P]),
    ("w8a8_smooth_rmsnorm_quant", _I, [_P, _P, _P, _P, _F, _I64, _I64, _P, _P, _P]),
    ("w8a8_silu_mul_quant", _I, [_P, _I64, _I64, _P, _P, _P]),
    ("w8a8_gemm_workspace_size", _SZ, [_I64, _I64, _I64]),
    ("w8a8_gemm_dequant", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]),
    ("w8a8_gemm_dequant_ex", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _SZ, _I, _I,
                                  _I, _P]),
    ("w8a8_gemm_workspace_size_ex", _SZ, [_I64, _I64, _I64, _I, _I, _I]),
    ("w8a8_gemm_dequant_noalloc", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    ("w8a8_gemm_silu_quant_workspace_size", _SZ, [_I64, _I64, _I64]),
    ("w8a8_gemm_silu_quant", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    ("w8a8_gemm_rmsnorm_quant_workspace_size", _SZ, [_I64, _I64, _I64]),
    ("w8a8_gemm_rmsnorm_quant_one_launch_ok", _I, [_I64, _I64, _I64]),
    ("w8a8_gemm_rmsnorm_quant", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _F, _P,
                                     _P, _P, _SZ, _P]),
    ("w8a8_gemm_rmsnorm_quant_ex", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _F,
                                        _P, _P, _P, _SZ, _I, _P]),
    ("w8a8_gemm_silu_quant_fp8_workspace_size", _SZ, [_I64, _I64, _I64]),
    ("w8a8_gemm_silu_quant_fp8", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ,
                                      _P]),
    ("w8a8_probe_i8_mma", _I, [C.c_longlong, _I, _I, _P]),
    ("w8a8_selftest_wait_timeout", _I, [C.c_ulonglong, _P]),
    ("w8a8_set_overlap", _I, [_I]),
    ("w8a8_get_overlap", _I, []),
    ("w8a8_device_status", _I, [_I]),
    ("w8a8_last_device_status", _I, [_P]),
    ("w8a8_status_string", C.c_char_p, [_I]),
    ("w8a8_version", _I, []),
    ("w8a8_quantize_rows_fp8", _I, [_P, _P, _I64, _I64, _P, _P, _P]),
    ("w8a8_smooth_rmsnorm_quant_fp8", _I, [_P, _P, _P, _P, _F, _I64, _I64, _P, _P, _P]),
    ("w8a8_silu_mul_quant_fp8", _I, [_P, _I64, _I64, _P, _P, _P]),
    ("w8a8_gemm_fp8_workspace_size", _SZ, [_I64, _I64, _I64, _I, _I, _I]),
    ("w8a8_gemm_dequant_fp8", _I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _SZ, _I, _I,
                                   _I, _P]),
    ("w8a8_gptq_workspace_size", _SZ, [_I64, _I64]),
    ("w8a8_block_decode_workspace_size", _SZ, [_I64, _I64, _I64, _I64]),
    ("w8a8_block_decode", _I, [_P, _P, _SZ, _P]),
    ("w8a8_probe_f64_fma", _I, [C.c_longlong, _I, _P, _P]),
    ("w8a8_gptq_quantize", _I, [_P, _P, _P, _I64, _I64, _I64, C.c_double, _P, _P, _P, _P, _SZ,
                                _P]),
]

# FP8 codes are OCP E4M3 bit patterns, carried in torch.float8_e4m3fn tensors
FP8 = torch.float8_e4m3fn

_lib = None
_lock = threading.Lock()


class W8A8Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def lib():
    """The loaded CUDA library. Fails loudly when it has not been built: there is no
    fallback implementation."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"{LIB_PATH} is missing; build it with "
                        "`python -m int8_w8a8_quantized_smoothed_b200.build`")
                L = C.CDLL(LIB_PATH)
                for name, res, args in SIGNATURES:
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


def _check(fn, rc):
    if rc != 0:
        raise W8A8Error(fn, rc)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def w8a8_status_string(status: int) -> str:
    return lib().w8a8_status_string(int(status)).decode()


def w8a8_version() -> int:
    return lib().w8a8_version()


def w8a8_selftest_wait_timeout(limit_ns: int = 5_000_000, stream=None) -> None:
    """Launch the failure-path self-test: two waits that nothing satisfies give up after
    limit_ns; the next w8a8_device_status() reports W8A8_ERR_TIMEOUT."""
    _check("w8a8_selftest_wait_timeout",
           lib().w8a8_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def w8a8_probe_i8_mma(iters: int, n: int = 256, ctas: int = 0, stream=None) -> None:
    """Measurement aid: back-to-back dense INT8 tcgen05 MMAs on every SM (not the W8A8 path)."""
    _check("w8a8_probe_i8_mma", lib().w8a8_probe_i8_mma(int(iters), int(n), int(ctas),
                                                         _stream(stream)))


def w8a8_set_overlap(mode: int) -> int:
    """0 plain stream order, 1 dependent launch (default), 2 also prefetch static weights
    before the dependency wait (weights must not be written by kernels still in flight).
    Returns the previous mode."""
    rc = lib().w8a8_set_overlap(int(mode))
    if rc < 0:
        raise W8A8Error("w8a8_set_overlap", rc)
    return rc


def w8a8_get_overlap() -> int:
    return lib().w8a8_get_overlap()


def w8a8_device_status(reset: bool = False) -> int:
    """Synchronizes the current device; returns 0 or -6 (a bounded wait ran out)."""
    return lib().w8a8_device_status(1 if reset else 0)


def w8a8_last_device_status(stream=None) -> int:
    """Waits for `stream` (default: the current stream) only; returns 0 or -6 (a bounded
    wait of a kernel on this device ran out; the word is not cleared)."""
    return lib().w8a8_last_device_status(_stream(stream))


def w8a8_quantize_rows(x, smooth_inv=None, q=None, s_tok=None, stream=None):
    """Per-token int8 quantization of bf16 x [M, K] (optionally x * smooth_inv)."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    if smooth_inv is not None:
        _need(smooth_inv, "smooth_inv", torch.float32, (K,))
    q = torch.empty((M, K), dtype=torch.int8, device=x.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(q, "q", torch.int8, (M, K))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_quantize_rows", lib().w8a8_quantize_rows(
        _ptr(x), _ptr(smooth_inv), M, K, _ptr(q), _ptr(s_tok), _stream(stream)))
    return q, s_tok


def w8a8_quantize_rows_static(x, scale, smooth_inv=None, q=None, s_tok=None, stream=None):
    """Static per-tensor int8 quantization of bf16 x [M, K] with a fixed calibrated scale;
    s_tok (filled with the scale) is returned too so that the GEMM can consume it."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    if smooth_inv is not None:
        _need(smooth_inv, "smooth_inv", torch.float32, (K,))
    q = torch.empty((M, K), dtype=torch.int8, device=x.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(q, "q", torch.int8, (M, K))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_quantize_rows_static", lib().w8a8_quantize_rows_static(
        _ptr(x), _ptr(smooth_inv), float(scale), M, K, _ptr(q), _ptr(s_tok), _stream(stream)))
    return q, s_tok


def w8a8_smooth_rmsnorm_quant(x, gamma_smoothed, eps, residual=None, h_out=None, q=None,
                              s_tok=None, stream=None):
    """RMSNorm with SmoothQuant-folded gamma, fused with per-token quantization.
    With `residual`, h = bf16(x + residual) is normalized and also returned."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    _need(gamma_smoothed, "gamma_smoothed", torch.float32, (K,))
    if residual is not None:
        _need(residual, "residual", torch.bfloat16, (M, K))
        h_out = torch.empty_like(x) if h_out is None else h_out
        _need(h_out, "h_out", torch.bfloat16, (M, K))
    q = torch.empty((M, K), dtype=torch.int8, device=x.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(q, "q", torch.int8, (M, K))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_smooth_rmsnorm_quant", lib().w8a8_smooth_rmsnorm_quant(
        _ptr(x), _ptr(residual), _ptr(h_out), _ptr(gamma_smoothed), float(eps), M, K, _ptr(q),
        _ptr(s_tok), _stream(stream)))
    if residual is not None:
        return q, s_tok, h_out
    return q, s_tok


def w8a8_silu_mul_quant(gate_up, q=None, s_tok=None, stream=None):
    """SiLU(gate) * up over the [M, 2I] gate|up halves, fused with per-token quantization."""
    _need(gate_up, "gate_up", torch.bfloat16)
    M, I2 = gate_up.shape
    if I2 % 2:
        raise ValueError("gate_up must have an even number of columns")
    I = I2 // 2
    q = torch.empty((M, I), dtype=torch.int8, device=gate_up.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=gate_up.device) if s_tok is None else s_tok
    _need(q, "q", torch.int8, (M, I))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_silu_mul_quant", lib().w8a8_silu_mul_quant(
        _ptr(gate_up), M, I, _ptr(q), _ptr(s_tok), _stream(stream)))
    return q, s_tok


def w8a8_quantize_rows_fp8(x, smooth_inv=None, q=None, s_tok=None, stream=None):
    """Per-token FP8 (E4M3, scale amax / 448) quantization of bf16 x [M, K]."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    if smooth_inv is not None:
        _need(smooth_inv, "smooth_inv", torch.float32, (K,))
    q = torch.empty((M, K), dtype=FP8, device=x.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(q, "q", FP8, (M, K))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_quantize_rows_fp8", lib().w8a8_quantize_rows_fp8(
        _ptr(x), _ptr(smooth_inv), M, K, _ptr(q), _ptr(s_tok), _stream(stream)))
    return q, s_tok


def w8a8_smooth_rmsnorm_quant_fp8(x, gamma_smoothed, eps, residual=None, h_out=None, q=None,
                                  s_tok=None, stream=None):
    """w8a8_smooth_rmsnorm_quant with FP8 (E4M3) codes."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    _need(gamma_smoothed, "gamma_smoothed", torch.float32, (K,))
    if residual is not None:
        _need(residual, "residual", torch.bfloat16, (M, K))
        h_out = torch.empty_like(x) if h_out is None else h_out
        _need(h_out, "h_out", torch.bfloat16, (M, K))
    q = torch.empty((M, K), dtype=FP8, device=x.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(q, "q", FP8, (M, K))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_smooth_rmsnorm_quant_fp8", lib().w8a8_smooth_rmsnorm_quant_fp8(
        _ptr(x), _ptr(residual), _ptr(h_out), _ptr(gamma_smoothed), float(eps), M, K, _ptr(q),
        _ptr(s_tok), _stream(stream)))
    if residual is not None:
        return q, s_tok, h_out
    return q, s_tok


def w8a8_silu_mul_quant_fp8(gate_up, q=None, s_tok=None, stream=None):
    """w8a8_silu_mul_quant with FP8 (E4M3) codes."""
    _need(gate_up, "gate_up", torch.bfloat16)
    M, I2 = gate_up.shape
    if I2 % 2:
        raise ValueError("gate_up must have an even number of columns")
    I = I2 // 2
    q = torch.empty((M, I), dtype=FP8, device=gate_up.device) if q is None else q
    s_tok = torch.empty(M, dtype=torch.float32, device=gate_up.device) if s_tok is None else s_tok
    _need(q, "q", FP8, (M, I))
    _need(s_tok, "s_tok", torch.float32, (M,))
    _check("w8a8_silu_mul_quant_fp8", lib().w8a8_silu_mul_quant_fp8(
        _ptr(gate_up), M, I, _ptr(q), _ptr(s_tok), _stream(stream)))
    return q, s_tok


def w8a8_gemm_fp8_workspace_size(M, N, K, variant=0, ctas=0, tile_n=0) -> int:
    return int(lib().w8a8_gemm_fp8_workspace_size(M, N, K, variant, ctas, tile_n))


def w8a8_gemm_workspace_size(M, N, K) -> int:
    return int(lib().w8a8_gemm_workspace_size(M, N, K))


def w8a8_gemm_workspace_size_ex(M, N, K, variant=0, ctas=0, tile_n=0) -> int:
    return int(lib().w8a8_gemm_workspace_size_ex(M, N, K, variant, ctas, tile_n))


class Workspace:
    """A zero-filled device workspace that grows on demand (the library never allocates).
    One instance serves calls issued in order on one stream."""

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.buf = None

    def get(self, nbytes):
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=self.device)
        return self.buf, self.buf.numel()


_default_ws = {}


def _workspace_for(device):
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(device)
    return ws


def w8a8_gemm_dequant_ex(xq, s_tok, wq, s_ch, y=None, acc_out=None, workspace=None,
                         variant=0, ctas=0, tile_n=0, stream=None):
    """y = bf16((float(xq @ wq.T) * s_tok[:, None]) * s_ch[None, :]) on the tensor cores.
    variant 0 = automatic, 1 = persistent tile kernel, 2 = swap-AB stream-K kernel
    (ctas = persistent CTAs, 0 = one per SM)."""
    _need(xq, "xq", torch.int8)
    _need(wq, "wq", torch.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"xq [M,K] and wq [N,K] disagree on K: {K} vs {K2}")
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch, "s_ch", torch.float32, (N,))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N))
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.int32, (M, N))
    need = w8a8_gemm_workspace_size_ex(M, N, K, variant, ctas, tile_n)
    if workspace is None:
        workspace = _workspace_for(xq.device)
    if isinstance(workspace, Workspace):
        wbuf, wbytes = workspace.get(need)
    else:
        wbuf, wbytes = workspace, (0 if workspace is None else workspace.numel()
                                   * workspace.element_size())
    _check("w8a8_gemm_dequant", lib().w8a8_gemm_dequant_ex(
        _ptr(xq), _ptr(s_tok), _ptr(wq), _ptr(s_ch), M, N, K, _ptr(y), _ptr(acc_out),
        _ptr(wbuf), wbytes, int(variant), int(ctas), int(tile_n), _stream(stream)))
    return y


def w8a8_gemm_dequant_fp8(xq, s_tok, wq, s_ch, y=None, acc_out=None, workspace=None,
                          variant=0, ctas=0, tile_n=0, stream=None):
    """FP8 GEMM: y = bf16((acc * s_tok[:, None]) * s_ch[None, :]) with acc the binary32
    tensor-core sum of E4M3 products (xq [M, K], wq [N, K] as torch.float8_e4m3fn).
    variant 0 = automatic, 1 = persistent tile kernel, 2 = swap-AB stream-K kernel."""
    _need(xq, "xq", FP8)
    _need(wq, "wq", FP8)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"xq [M,K] and wq [N,K] disagree on K: {K} vs {K2}")
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch, "s_ch", torch.float32, (N,))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N))
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.float32, (M, N))
    need = w8a8_gemm_fp8_workspace_size(M, N, K, variant, ctas, tile_n)
    if workspace is None:
        workspace = _workspace_for(xq.device)
    if isinstance(workspace, Workspace):
        wbuf, wbytes = workspace.get(need)
    else:
        wbuf, wbytes = workspace, (0 if workspace is None else workspace.numel()
                                   * workspace.element_size())
    _check("w8a8_gemm_dequant_fp8", lib().w8a8_gemm_dequant_fp8(
        _ptr(xq), _ptr(s_tok), _ptr(wq), _ptr(s_ch), M, N, K, _ptr(y), _ptr(acc_out),
        _ptr(wbuf), wbytes, int(variant), int(ctas), int(tile_n), _stream(stream)))
    return y


def w8a8_gemm_dequant(xq, s_tok, wq, s_ch, y=None, acc_out=None, workspace=None, stream=None):
    return w8a8_gemm_dequant_ex(xq, s_tok, wq, s_ch, y=y, acc_out=acc_out,
                                workspace=workspace, stream=stream)


def w8a8_gemm_silu_quant_workspace_size(M: int, I: int, K: int) -> int:
    return int(lib().w8a8_gemm_silu_quant_workspace_size(M, I, K))


def w8a8_gemm_silu_quant(xq, s_tok, wq_il, s_ch_il, a=None, q=None, s_out=None,
                         workspace=None, stream=None):
    """The gate|up GEMM with the SiLU(gate)*up epilogue, then per-token quantization of a:
    the same q, s as w8a8_gemm_dequant + w8a8_silu_mul_quant on the plain weight. wq_il,
    s_ch_il: the gate|up weight and scales with rows interleaved in blocks of 64 (see
    prep.interleave_gate_up). Returns (q, s_out, a)."""
    _need(xq, "xq", torch.int8)
    _need(wq_il, "wq_il", torch.int8)
    M, K = xq.shape
    N, K2 = wq_il.shape
    if K != K2 or N % 2:
        raise ValueError(f"xq [M,K] and wq_il [2I,K] disagree: {tuple(xq.shape)} {tuple(wq_il.shape)}")
    I = N // 2
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch_il, "s_ch_il", torch.float32, (N,))
    e = dict(device=xq.device)
    a = torch.empty((M, I), dtype=torch.float32, **e) if a is None else a
    q = torch.empty((M, I), dtype=torch.int8, **e) if q is None else q
    s_out = torch.empty(M, dtype=torch.float32, **e) if s_out is None else s_out
    _need(a, "a", torch.float32, (M, I))
    _need(q, "q", torch.int8, (M, I))
    _need(s_out, "s_out", torch.float32, (M,))
    need = w8a8_gemm_silu_quant_workspace_size(M, I, K)
    if workspace is None:
        workspace = _workspace_for(xq.device)
    if isinstance(workspace, Workspace):
        wbuf, wbytes = workspace.get(need)
    else:
        wbuf, wbytes = workspace, (0 if workspace is None else workspace.numel()
                                   * workspace.element_size())
    _check("w8a8_gemm_silu_quant", lib().w8a8_gemm_silu_quant(
        _ptr(xq), _ptr(s_tok), _ptr(wq_il), _ptr(s_ch_il), M, I, K, _ptr(a), _ptr(q),
        _ptr(s_out), _ptr(wbuf), wbytes, _stream(stream)))
    return q, s_out, a


def w8a8_gemm_rmsnorm_quant_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().w8a8_gemm_rmsnorm_quant_workspace_size(M, N, K))


def w8a8_gemm_rmsnorm_quant_one_launch_ok(M: int, N: int, K: int) -> bool:
    """Whether the one-launch form (the GEMM with the RMSNorm tail) applies to the shape."""
    return bool(lib().w8a8_gemm_rmsnorm_quant_one_launch_ok(M, N, K))


def w8a8_gemm_rmsnorm_quant(xq, s_tok, wq, s_ch, residual, gamma_smoothed, eps, y=None,
                            h_out=None, q=None, s_out=None, workspace=None, one_launch=False,
                            stream=None):
    """The GEMM + dequant into y, then h = bf16(y + residual) and the smoothed RMSNorm of h
    with per-token quantization: the same y, h, q, s as w8a8_gemm_dequant followed by
    w8a8_smooth_rmsnorm_quant(y, ..., residual=residual). h_out may be residual (in place).
    one_launch: the GEMM's last CTAs run the row pass (decode sizes only) instead of a second
    launch. Returns (q, s_out, h_out, y)."""
    _need(xq, "xq", torch.int8)
    _need(wq, "wq", torch.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"xq [M,K] and wq [N,K] disagree: {tuple(xq.shape)} {tuple(wq.shape)}")
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch, "s_ch", torch.float32, (N,))
    _need(residual, "residual", torch.bfloat16, (M, N))
    _need(gamma_smoothed, "gamma_smoothed", torch.float32, (N,))
    e = dict(device=xq.device)
    y = torch.empty((M, N), dtype=torch.bfloat16, **e) if y is None else y
    h_out = torch.empty((M, N), dtype=torch.bfloat16, **e) if h_out is None else h_out
    q = torch.empty((M, N), dtype=torch.int8, **e) if q is None else q
    s_out = torch.empty(M, dtype=torch.float32, **e) if s_out is None else s_out
    _need(y, "y", torch.bfloat16, (M, N))
    _need(h_out, "h_out", torch.bfloat16, (M, N))
    _need(q, "q", torch.int8, (M, N))
    _need(s_out, "s_out", torch.float32, (M,))
    need = w8a8_gemm_rmsnorm_quant_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace_for(xq.device)
    if isinstance(workspace, Workspace):
        wbuf, wbytes = workspace.get(need)
    else:
        wbuf, wbytes = workspace, (0 if workspace is None else workspace.numel()
                                   * workspace.element_size())
    _check("w8a8_gemm_rmsnorm_quant_ex", lib().w8a8_gemm_rmsnorm_quant_ex(
        _ptr(xq), _ptr(s_tok), _ptr(wq), _ptr(s_ch), M, N, K, _ptr(y), _ptr(residual),
        _ptr(h_out), _ptr(gamma_smoothed), float(eps), _ptr(q), _ptr(s_out), _ptr(wbuf), wbytes,
        1 if one_launch else 0, _stream(stream)))
    return q, s_out, h_out, y


def w8a8_gemm_silu_quant_fp8_workspace_size(M: int, I: int, K: int) -> int:
    return int(lib().w8a8_gemm_silu_quant_fp8_workspace_size(M, I, K))


def w8a8_gemm_silu_quant_fp8(xq, s_tok, wq_il, s_ch_il, a=None, q=None, s_out=None,
                             workspace=None, stream=None):
    """w8a8_gemm_silu_quant with FP8 operands and codes (xq, wq_il, q as
    torch.float8_e4m3fn; s_out = max |a| / 448). Returns (q, s_out, a)."""
    _need(xq, "xq", FP8)
    _need(wq_il, "wq_il", FP8)
    M, K = xq.shape
    N, K2 = wq_il.shape
    if K != K2 or N % 2:
        raise ValueError(f"xq [M,K] and wq_il [2I,K] disagree: {tuple(xq.shape)} {tuple(wq_il.shape)}")
    I = N // 2
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch_il, "s_ch_il", torch.float32, (N,))
    e = dict(device=xq.device)
    a = torch.empty((M, I), dtype=torch.float32, **e) if a is None else a
    q = torch.empty((M, I), dtype=FP8, **e) if q is None else q
    s_out = torch.empty(M, dtype=torch.float32, **e) if s_out is None else s_out
    _need(a, "a", torch.float32, (M, I))
    _need(q, "q", FP8, (M, I))
    _need(s_out, "s_out", torch.float32, (M,))
    need = w8a8_gemm_silu_quant_fp8_workspace_size(M, I, K)
    if workspace is None:
        workspace = _workspace_for(xq.device)
    if isinstance(workspace, Workspace):
        wbuf, wbytes = workspace.get(need)
    else:
        wbuf, wbytes = workspace, (0 if workspace is None else workspace.numel()
                                   * workspace.element_size())
    _check("w8a8_gemm_silu_quant_fp8", lib().w8a8_gemm_silu_quant_fp8(
        _ptr(xq), _ptr(s_tok), _ptr(wq_il), _ptr(s_ch_il), M, I, K, _ptr(a), _ptr(q),
        _ptr(s_out), _ptr(wbuf), wbytes, _stream(stream)))
    return q, s_out, a


NOALLOC_SCRATCH_BYTES = 8 << 20  # W8A8_NOALLOC_SCRATCH_BYTES in include/w8a8.h


def w8a8_gemm_dequant_noalloc(xq, s_tok, wq, s_ch, y=None, stream=None):
    """The small-M (M <= 256) GEMM + dequant without any device allocation by the library:
    its stream-K scratch is a fixed 8 MiB array inside the library, for callers that cannot
    allocate (see include/w8a8.h). Only `y` is allocated here, and only if not given."""
    _need(xq, "xq", torch.int8)
    _need(wq, "wq", torch.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"xq [M,K] and wq [N,K] disagree on K: {K} vs {K2}")
    _need(s_tok, "s_tok", torch.float32, (M,))
    _need(s_ch, "s_ch", torch.float32, (N,))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N))
    _check("w8a8_gemm_dequant_noalloc", lib().w8a8_gemm_dequant_noalloc(
        _ptr(xq), _ptr(s_tok), _ptr(wq), _ptr(s_ch), M, N, K, _ptr(y), _stream(stream)))
    return y


def w8a8_probe_f64_fma(iters: int, ctas: int, out=None, stream=None):
    """Binary64 FMA throughput probe: 2 * 8 * iters * 256 * ctas flops. Returns out."""
    if out is None:
        out = torch.empty(ctas * 256, dtype=torch.float64, device="cuda")
    _check("w8a8_probe_f64_fma", lib().w8a8_probe_f64_fma(int(iters), int(ctas), _ptr(out),
                                                          _stream(stream)))
    return out


def w8a8_gptq_workspace_size(N: int, K: int) -> int:
    return int(lib().w8a8_gptq_workspace_size(N, K))


def w8a8_gptq_quantize(w, x_cal, smooth=None, damp=0.01, wq=None, s_ch=None, want_u=False,
                       workspace=None, stream=None):
    """GPTQ int8 weights (offline): w bf16 [N, K] (times smooth [K] if given), calibration
    inputs x_cal fp32 [T, K] as the layer receives them. Synchronizes the stream.
    Returns (wq int8 [N, K], s_ch fp32 [N]) and, with want_u, U fp64 [K, K]."""
    _need(w, "w", torch.bfloat16)
    N, K = w.shape
    _need(x_cal, "x_cal", torch.float32)
    T, K2 = x_cal.shape
    if K2 != K:
        raise ValueError(f"w [N,K] and x_cal [T,K] disagree on K: {K} vs {K2}")
    if smooth is not None:
        _need(smooth, "smooth", torch.float32, (K,))
    e = dict(device=w.device)
    wq = torch.empty((N, K), dtype=torch.int8, **e) if wq is None else wq
    s_ch = torch.empty(N, dtype=torch.float32, **e) if s_ch is None else s_ch
    _need(wq, "wq", torch.int8, (N, K))
    _need(s_ch, "s_ch", torch.float32, (N,))
    u = torch.empty((K, K), dtype=torch.float64, **e) if want_u else None
    need = w8a8_gptq_workspace_size(N, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, **e)
    _check("w8a8_gptq_quantize", lib().w8a8_gptq_quantize(
        _ptr(w), _ptr(smooth), _ptr(x_cal), N, K, T, float(damp), _ptr(wq), _ptr(s_ch),
        _ptr(u), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return (wq, s_ch, u) if want_u else (wq, s_ch)


class _Linear(C.Structure):
    _fields_ = [("wq", C.c_void_p), ("s_ch", C.c_void_p)]


class _BlockIO(C.Structure):
    """Mirror of w8a8_block_io (include/w8a8.h)."""
    _fields_ = [("M", C.c_int64), ("H", C.c_int64), ("I", C.c_int64), ("QKV", C.c_int64),
                ("eps", C.c_float),
                ("x", C.c_void_p), ("attn", C.c_void_p),
                ("gamma1", C.c_void_p), ("sinv_o", C.c_void_p), ("gamma2", C.c_void_p),
                ("qkv", _Linear), ("o", _Linear), ("gate_up_il", _Linear), ("down", _Linear),
                ("qkv_out", C.c_void_p), ("o_out", C.c_void_p), ("h_out", C.c_void_p),
                ("y_out", C.c_void_p), ("a_out", C.c_void_p),
                ("q1", C.c_void_p), ("q2", C.c_void_p), ("q3", C.c_void_p), ("q4", C.c_void_p),
                ("s1", C.c_void_p), ("s2", C.c_void_p), ("s3", C.c_void_p), ("s4", C.c_void_p)]


def w8a8_block_decode_workspace_size(M, H, I, QKV) -> int:
    return int(lib().w8a8_block_decode_workspace_size(M, H, I, QKV))


class BlockBuffers:
    """Outputs and intermediates of one fused decoder-block call (allocated once, reused)."""

    def __init__(self, M, H, I, QKV, device):
        e = dict(device=device)
        self.qkv = torch.empty((M, QKV), dtype=torch.bfloat16, **e)
        self.o = torch.empty((M, H), dtype=torch.bfloat16, **e)
        self.h = torch.empty((M, H), dtype=torch.bfloat16, **e)
        self.y = torch.empty((M, H), dtype=torch.bfloat16, **e)
        self.a = torch.empty((M, I), dtype=torch.float32, **e)
        self.q = [torch.empty((M, H), dtype=torch.int8, **e) for _ in range(3)] + \
                 [torch.empty((M, I), dtype=torch.int8, **e)]
        self.s = [torch.empty(M, dtype=torch.float32, **e) for _ in range(4)]
        need = w8a8_block_decode_workspace_size(M, H, I, QKV)
        self.workspace = torch.zeros(max(need, 256), dtype=torch.uint8, **e)


def w8a8_block_decode(x, attn, gamma1, sinv_o, gamma2, qkv, o, gate_up_il, down, eps,
                      buffers=None, stream=None):
    """One decoder block's linear path at decode sizes in a single persistent kernel.
    qkv, o, gate_up_il, down: (wq int8 [N, K], s_ch fp32 [N]) with gate_up_il interleaved as
    for w8a8_gemm_silu_quant. Returns the BlockBuffers (y = the down projection's output)."""
    _need(x, "x", torch.bfloat16)
    M, H = x.shape
    _need(attn, "attn", torch.bfloat16, (M, H))
    for t, n in ((gamma1, "gamma1"), (sinv_o, "sinv_o"), (gamma2, "gamma2")):
        _need(t, n, torch.float32, (H,))
    QKV = qkv[0].shape[0]
    I = down[0].shape[1]
    for (wq, sc), n, shape in ((qkv, "qkv", (QKV, H)), (o, "o", (H, H)),
                               (gate_up_il, "gate_up_il", (2 * I, H)), (down, "down", (H, I))):
        _need(wq, n + ".wq", torch.int8, shape)
        _need(sc, n + ".s_ch", torch.float32, (shape[0],))
    b = BlockBuffers(M, H, I, QKV, x.device) if buffers is None else buffers
    io = _BlockIO(M=M, H=H, I=I, QKV=QKV, eps=float(eps),
                  x=x.data_ptr(), attn=attn.data_ptr(), gamma1=gamma1.data_ptr(),
                  sinv_o=sinv_o.data_ptr(), gamma2=gamma2.data_ptr(),
                  qkv=_Linear(qkv[0].data_ptr(), qkv[1].data_ptr()),
                  o=_Linear(o[0].data_ptr(), o[1].data_ptr()),
                  gate_up_il=_Linear(gate_up_il[0].data_ptr(), gate_up_il[1].data_ptr()),
                  down=_Linear(down[0].data_ptr(), down[1].data_ptr()),
                  qkv_out=b.qkv.data_ptr(), o_out=b.o.data_ptr(), h_out=b.h.data_ptr(),
                  y_out=b.y.data_ptr(), a_out=b.a.data_ptr(),
                  q1=b.q[0].data_ptr(), q2=b.q[1].data_ptr(), q3=b.q[2].data_ptr(),
                  q4=b.q[3].data_ptr(), s1=b.s[0].data_ptr(), s2=b.s[1].data_ptr(),
                  s3=b.s[2].data_ptr(), s4=b.s[3].data_ptr())
    _check("w8a8_block_decode", lib().w8a8_block_decode(
        C.byref(io), _ptr(b.workspace), b.workspace.numel(), _stream(stream)))
    return b
