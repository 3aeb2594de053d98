"""The C-ABI library loads and exports every entry point include/w8a8.h declares; host-side
argument validation answers before any device work (these run without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import pytest

import int8_w8a8_quantized_smoothed_b200 as w8
from int8_w8a8_quantized_smoothed_b200 import build as w8build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a8.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"W8A8_API\s+[\w\s\*]+?\b(w8a8_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def L():
    w8build.build()
    return w8.lib()


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("w8a8_smooth_rmsnorm_quant", "w8a8_quantize_rows", "w8a8_gemm_dequant",
              "w8a8_silu_mul_quant", "w8a8_gemm_workspace_size", "w8a8_device_status",
              "w8a8_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", w8.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(w8a8_\w+)", out))
    declared = set(declared_functions())
    assert declared <= exported, declared - exported
    assert {s[0] for s in w8.SIGNATURES} == declared
    for n in declared:
        assert getattr(L, n) is not None


def test_status_strings_and_version(L):
    assert L.w8a8_status_string(0) == b"ok"
    assert b"aligned" in L.w8a8_status_string(-2)
    assert L.w8a8_status_string(12345) == b"unknown status"
    assert L.w8a8_version() >> 16 == 1


def _p(v):
    return C.c_void_p(v)


A = 0x10000  # a 16-byte aligned fake address; never dereferenced by the host checks


def test_host_validation_without_device(L):
    # null pointers / bad sizes / misalignment are rejected before any CUDA call
    assert L.w8a8_quantize_rows(None, None, 4, 64, _p(A), _p(A), None) == -1
    assert L.w8a8_quantize_rows(_p(A), None, 0, 64, _p(A + 4096), _p(A), None) == -1
    assert L.w8a8_quantize_rows(_p(A), None, 4, 24, _p(A + 4096), _p(A), None) == -3
    assert L.w8a8_quantize_rows(_p(A), None, 4, 65536, _p(A + 4096), _p(A), None) == -3
    assert L.w8a8_quantize_rows(_p(A + 2), None, 4, 64, _p(A + 4096), _p(A), None) == -2
    assert L.w8a8_quantize_rows(_p(A), None, 4, 64, _p(A), _p(A + 8192), None) == -1
    # residual without h_out
    assert L.w8a8_smooth_rmsnorm_quant(_p(A), _p(A + 4096), None, _p(A), C.c_float(1e-5), 4, 64,
                                       _p(A), _p(A), None) == -1
    assert L.w8a8_smooth_rmsnorm_quant(_p(A), None, None, _p(A), C.c_float(-1.0), 4, 64,
                                       _p(A), _p(A), None) == -1
    assert L.w8a8_silu_mul_quant(_p(A), 4, 40, _p(A), _p(A), None) == -3
    # static scale: must be finite and positive; same shape / alignment rules
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert L.w8a8_quantize_rows_static(_p(A), None, C.c_float(bad), 4, 64, _p(A + 4096),
                                           None, None) == -1
    assert L.w8a8_quantize_rows_static(_p(A), None, C.c_float(0.1), 4, 24, _p(A + 4096), None,
                                       None) == -3
    assert L.w8a8_quantize_rows_static(_p(A), _p(A + 4), C.c_float(0.1), 4, 64, _p(A + 4096),
                                       None, None) == -2
    # GEMM: N % 8, K % 16, K limit, alignment
    args = [_p(A), _p(A), _p(A), _p(A)]
    assert L.w8a8_gemm_dequant(*args, 4, 12, 64, _p(A), None, None, 0, None) == -3
    assert L.w8a8_gemm_dequant(*args, 4, 16, 40, _p(A), None, None, 0, None) == -3
    assert L.w8a8_gemm_dequant(*args, 4, 16, 133152, _p(A), None, None, 0, None) == -3
    assert L.w8a8_gemm_dequant(*args, 0, 16, 64, _p(A), None, None, 0, None) == -1
    assert L.w8a8_gemm_dequant(_p(A), _p(A), _p(A + 8), _p(A), 4, 16, 64, _p(A), None, None, 0,
                               None) == -2
    assert L.w8a8_gemm_dequant(None, _p(A), _p(A), _p(A), 4, 16, 64, _p(A), None, None, 0,
                               None) == -1
    assert L.w8a8_gemm_workspace_size(4, 12, 64) == 0


def test_valid_call_without_gpu_reports_no_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.w8a8_quantize_rows(_p(A), None, 4, 64, _p(A + 4096), _p(A + 8192), None) == -7
    assert L.w8a8_device_status(0) == -7


def test_gemm_rmsnorm_quant_host_checks(L):
    # the o projection + residual RMSNorm entry point: argument checks, then the device
    Y, R, H, G, Q, S, W = (_p(A + i * 0x100000) for i in range(7))
    ws = 1 << 20

    def call(M=4, N=1024, K=512, y=Y, res=R, h=H, eps=1e-5, one=0, wbytes=ws, g=G):
        return L.w8a8_gemm_rmsnorm_quant_ex(_p(A), _p(A), _p(A), _p(A), M, N, K, y, res, h, g,
                                            C.c_float(eps), Q, S, W, wbytes, one, None)

    assert call(g=None) == -1                      # a null pointer
    assert call(eps=-1.0) == -1                    # eps < 0
    assert call(eps=float("nan")) == -1
    assert call(one=2) == -1                       # the form selector
    assert call(y=R) == -1                         # y may not alias the residual ...
    assert call(h=Y) == -1                         # ... nor h_out
    assert call(N=1032) == -3                      # rows of N % 16 != 0
    assert call(K=40) == -3                        # the GEMM's K % 16
    assert call(h=_p(A + 0x600008)) == -2          # a misaligned output
    import torch
    if not torch.cuda.is_available():
        assert call() == -7                        # valid: no device here
        assert call(h=R) == -7                     # h_out may alias the residual


def test_gemm_rmsnorm_quant_one_launch_plan(L):
    # the one-launch form is the cluster split-K plan (M <= 64, few channel blocks, N <= 8192)
    ok = L.w8a8_gemm_rmsnorm_quant_one_launch_ok
    assert ok(1, 4096, 4096) == 1 and ok(64, 4096, 4096) == 1 and ok(5, 8192, 1024) == 1
    assert ok(65, 4096, 4096) == 0                 # tile kernels
    assert ok(4, 12288, 512) == 0                  # rows wider than 8192
    assert ok(3, 1024, 128) == 0                   # one k-block: the stream-K plan
    assert ok(4, 1032, 512) == 0                   # invalid row length
    assert L.w8a8_gemm_rmsnorm_quant_workspace_size(16, 4096, 4096) >= 4096
    assert L.w8a8_gemm_rmsnorm_quant_workspace_size(4, 1032, 512) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        w8.w8a8_quantize_rows(x)
