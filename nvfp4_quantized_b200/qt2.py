"""Thin ctypes binding of the qt2 C ABI (include/qt2.h).

Argument marshalling only: every function below forwards to the entry point of the same name
in ``libqt2.so`` (device pointers from torch tensors, the current CUDA stream) and raises
``QT2Error`` on a non-OK status.  There is no CPU or PyTorch fallback: if the library is
missing the import of any call fails loudly.  PyTorch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# QT2_LIBRARY=checked loads the checked build (every kernel store checked against its output
# array, include/qt2.h); anything else, or unset, the product library
LIB_PATH = os.path.join(_PKG, "libqt2_checked.so" if os.environ.get("QT2_LIBRARY") == "checked" else "libqt2.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "qt2.h")

QT2_OK = 0
QT2_ERR_INVALID_ARG, QT2_ERR_SHAPE, QT2_ERR_ALIGN, QT2_ERR_WORKSPACE = -1, -2, -3, -4
QT2_ERR_CUDA, QT2_ERR_TIMEOUT, QT2_ERR_DEVICE, QT2_ERR_NONFINITE, QT2_ERR_BOUNDS = -5, -6, -7, -8, -9
QT2_LAYOUT_ROW, QT2_LAYOUT_COL, QT2_LAYOUT_BOTH = 1, 2, 3
QT2_DTYPE_BF16, QT2_DTYPE_F32 = 0, 1
QT2_TID_SIGNS, QT2_TID_DY_ROW, QT2_TID_DY_COL, QT2_TID_W_COL, QT2_TID_X_COL = 0, 1, 2, 3, 4


class QT2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


# qt2_set_fault_hook: int hook(const char *site, void *user); 0 = proceed, 1 = fail, 2 = skip
FAULT_NONE, FAULT_FAIL, FAULT_SKIP = 0, 1, 2
FaultHookC = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_char_p, ctypes.c_void_p)


class NVFP4ViewC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libqt2.so (built in-tree by nvfp4_quantized_b200.build); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_quantized_b200.build` "
                                   "(there is no fallback path)")
            L = ctypes.CDLL(LIB_PATH)
            i32, i64, u32, u64, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t
            vp, f32 = ctypes.c_void_p, ctypes.c_float
            pv = ctypes.POINTER(NVFP4ViewC)
            psz = ctypes.POINTER(ctypes.c_size_t)
            sigs = {
                "qt2_version": (i32, []),
                "qt2_status_string": (ctypes.c_char_p, [i32]),
                "qt2_device_status": (i32, [vp, ctypes.POINTER(ctypes.c_int)]),
                "qt2_quant_fwd46_workspace_size": (i32, [i64, i64, psz]),
                "qt2_quant_fwd46": (i32, [vp, i64, i64, i64, i32, pv, pv, vp, sz, vp]),
                "qt2_quant_msedEN_workspace_size": (i32, [i64, i64, i32, psz]),
                "qt2_quant_msedEN": (i32, [vp, i64, i64, i64, i32, u64, u32, u32, pv, pv, vp, sz, vp]),
                "qt2_quant_msedEN_noalloc": (i32, [vp, i64, i64, i64, i32, u64, u32, u32, pv, pv, vp]),
                "qt2_quant_sr_workspace_size": (i32, [i64, i64, i32, psz]),
                "qt2_quant_sr": (i32, [vp, i64, i64, i64, i32, u64, u32, u32, pv, pv, vp, sz, vp]),
                "qt2_gemm_nvfp4": (i32, [pv, pv, i64, i64, i64, f32, vp, i32, i64, vp]),
                "qt2_linear_fwd_workspace_size": (i32, [i64, i64, i64, psz]),
                "qt2_linear_fwd": (i32, [vp, vp, i64, i64, i64, vp, vp, sz, vp]),
                "qt2_linear_bwd_workspace_size": (i32, [i64, i64, i64, psz]),
                "qt2_linear_bwd": (i32, [vp, vp, vp, i64, i64, i64, u64, vp, vp, i32, vp, sz, vp]),
                "qt2_quant_fwd46_local": (i32, [vp, i64, i64, i64, pv, vp]),
                "qt2_selftest_wait_timeout": (i32, [vp]),
                "qt2_set_fault_hook": (None, [FaultHookC, vp]),
                "qt2_selftest_division": (i32, [u32, u32, vp, vp]),
                "qt2_build_checked": (i32, []),
                "qt2_selftest_bounds": (i32, [vp]),
                "qt2_gemm_nvfp4_local": (i32, [pv, pv, i64, i64, i64, f32, vp, i32, i64, vp]),
                "qt2_quant_fwd46_sq_workspace_size": (i32, [i64, i64, psz]),
                "qt2_quant_fwd46_sq": (i32, [vp, i64, i64, i64, pv, pv, vp, sz, vp]),
                "qt2_quant_fwd46_msedEN_col_workspace_size": (i32, [i64, i64, psz]),
                "qt2_quant_fwd46_msedEN_col": (i32, [vp, i64, i64, i64, u64, u32, pv, pv, vp, sz, vp]),
                "qt2_linear_bwd_views_workspace_size": (i32, [i64, i64, i64, psz]),
                "qt2_linear_bwd_views": (i32, [vp, i64, i64, i64, u64, pv, pv, vp, vp, i32, vp, sz, vp]),
            }
            for name, (res, args) in sigs.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/qt2.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qt2_[A-Za-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    try:
        return lib().qt2_status_string(status).decode()
    except Exception:
        return "?"


def _check(fn: str, status: int):
    if status != QT2_OK:
        raise QT2Error(fn, status)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------------------------------------- views
@dataclass
class View:
    """An NVFP4 view in device memory: codes [R, C/2] uint8, scales [R*C/16] uint8 (tensor-core
    scale-factor order), tensor_scale [1] float32."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor

    @property
    def shape(self):
        return self.codes.shape[0], self.codes.shape[1] * 2

    def c(self) -> NVFP4ViewC:
        return NVFP4ViewC(self.codes.data_ptr(), self.scales.data_ptr(), self.tensor_scale.data_ptr())


def alloc_view(R: int, C: int, device="cuda") -> View:
    return View(torch.empty((R, C // 2), dtype=torch.uint8, device=device),
                torch.empty((R * C // 16,), dtype=torch.uint8, device=device),
                torch.empty((1,), dtype=torch.float32, device=device))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device buffer (torch's caching allocator aligns to at least 512)."""
    t = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t


# --------------------------------------------------------------------------------------------- entry points
def qt2_version() -> int:
    return lib().qt2_version()


def qt2_status_string(status: int) -> str:
    return status_string(status)


def qt2_device_status(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("qt2_device_status", lib().qt2_device_status(_stream(stream), ctypes.byref(code)))
    return code.value


def qt2_quant_fwd46_workspace_size(rows: int, cols: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_quant_fwd46_workspace_size", lib().qt2_quant_fwd46_workspace_size(rows, cols, ctypes.byref(n)))
    return n.value


def qt2_quant_fwd46(x: torch.Tensor, rows: int, cols: int, ld: int, layout_mask: int, row_out: View | None,
                    col_out: View | None, workspace: torch.Tensor, ws_bytes: int, stream=None) -> None:
    r = row_out.c() if row_out is not None else None
    c = col_out.c() if col_out is not None else None
    _check("qt2_quant_fwd46", lib().qt2_quant_fwd46(
        _ptr(x), rows, cols, ld, layout_mask, ctypes.byref(r) if r else None, ctypes.byref(c) if c else None,
        _ptr(workspace), ws_bytes, _stream(stream)))


def qt2_quant_msedEN_workspace_size(rows: int, cols: int, layout_mask: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_quant_msedEN_workspace_size",
           lib().qt2_quant_msedEN_workspace_size(rows, cols, layout_mask, ctypes.byref(n)))
    return n.value


def qt2_quant_msedEN(x: torch.Tensor, rows: int, cols: int, ld: int, layout_mask: int, seed: int,
                     tensor_id_row: int, tensor_id_col: int, row_out: View | None, col_out: View | None,
                     workspace: torch.Tensor, ws_bytes: int, stream=None) -> None:
    r = row_out.c() if row_out is not None else None
    c = col_out.c() if col_out is not None else None
    _check("qt2_quant_msedEN", lib().qt2_quant_msedEN(
        _ptr(x), rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
        ctypes.byref(r) if r else None, ctypes.byref(c) if c else None, _ptr(workspace), ws_bytes, _stream(stream)))


def qt2_quant_msedEN_noalloc(x: torch.Tensor, rows: int, cols: int, ld: int, layout_mask: int, seed: int,
                             tensor_id_row: int, tensor_id_col: int, row_out: View | None, col_out: View | None,
                             stream=None) -> None:
    """qt2_quant_msedEN without a workspace: the library's built-in scratch array is used
    (see include/qt2.h for its size limit and the rule that calls must not overlap)."""
    r = row_out.c() if row_out is not None else None
    c = col_out.c() if col_out is not None else None
    _check("qt2_quant_msedEN_noalloc", lib().qt2_quant_msedEN_noalloc(
        _ptr(x), rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
        ctypes.byref(r) if r else None, ctypes.byref(c) if c else None, _stream(stream)))


def qt2_quant_sr_workspace_size(rows: int, cols: int, layout_mask: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_quant_sr_workspace_size", lib().qt2_quant_sr_workspace_size(rows, cols, layout_mask, ctypes.byref(n)))
    return n.value


def qt2_quant_sr(x: torch.Tensor, rows: int, cols: int, ld: int, layout_mask: int, seed: int, tensor_id_row: int,
                 tensor_id_col: int, row_out: View | None, col_out: View | None, workspace: torch.Tensor,
                 ws_bytes: int, stream=None) -> None:
    r = row_out.c() if row_out is not None else None
    c = col_out.c() if col_out is not None else None
    _check("qt2_quant_sr", lib().qt2_quant_sr(
        _ptr(x), rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
        ctypes.byref(r) if r else None, ctypes.byref(c) if c else None, _ptr(workspace), ws_bytes, _stream(stream)))


def qt2_gemm_nvfp4(a: View, b: View, M: int, N: int, K: int, alpha: float, c: torch.Tensor, c_dtype: int,
                   ldc: int, stream=None) -> None:
    ac, bc = a.c(), b.c()
    _check("qt2_gemm_nvfp4", lib().qt2_gemm_nvfp4(ctypes.byref(ac), ctypes.byref(bc), M, N, K, alpha, _ptr(c),
                                                  c_dtype, ldc, _stream(stream)))


def qt2_linear_fwd_workspace_size(M: int, K: int, N: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_linear_fwd_workspace_size", lib().qt2_linear_fwd_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def qt2_linear_fwd(x: torch.Tensor, w: torch.Tensor, M: int, K: int, N: int, y: torch.Tensor,
                   workspace: torch.Tensor, ws_bytes: int, stream=None) -> None:
    _check("qt2_linear_fwd", lib().qt2_linear_fwd(_ptr(x), _ptr(w), M, K, N, _ptr(y), _ptr(workspace), ws_bytes,
                                                  _stream(stream)))


def qt2_linear_bwd_workspace_size(M: int, K: int, N: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_linear_bwd_workspace_size", lib().qt2_linear_bwd_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def qt2_linear_bwd(dy: torch.Tensor, x: torch.Tensor, w: torch.Tensor, M: int, K: int, N: int, seed: int,
                   dx: torch.Tensor, dw: torch.Tensor, dw_dtype: int, workspace: torch.Tensor, ws_bytes: int,
                   stream=None) -> None:
    _check("qt2_linear_bwd", lib().qt2_linear_bwd(_ptr(dy), _ptr(x), _ptr(w), M, K, N, seed, _ptr(dx), _ptr(dw),
                                                  dw_dtype, _ptr(workspace), ws_bytes, _stream(stream)))


def qt2_quant_fwd46_msedEN_col_workspace_size(rows: int, cols: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_quant_fwd46_msedEN_col_workspace_size",
           lib().qt2_quant_fwd46_msedEN_col_workspace_size(rows, cols, ctypes.byref(n)))
    return n.value


def qt2_quant_fwd46_msedEN_col(x: torch.Tensor, rows: int, cols: int, ld: int, seed: int, tensor_id_col: int,
                               row_out: View, col_out: View, workspace: torch.Tensor, ws_bytes: int,
                               stream=None) -> None:
    r, c = row_out.c(), col_out.c()
    _check("qt2_quant_fwd46_msedEN_col", lib().qt2_quant_fwd46_msedEN_col(
        _ptr(x), rows, cols, ld, seed, tensor_id_col, ctypes.byref(r), ctypes.byref(c), _ptr(workspace), ws_bytes,
        _stream(stream)))


def qt2_linear_bwd_views_workspace_size(M: int, K: int, N: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_linear_bwd_views_workspace_size", lib().qt2_linear_bwd_views_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def qt2_linear_bwd_views(dy: torch.Tensor, M: int, K: int, N: int, seed: int, x_col: View, w_col: View,
                         dx: torch.Tensor, dw: torch.Tensor, dw_dtype: int, workspace: torch.Tensor, ws_bytes: int,
                         stream=None) -> None:
    xc, wc = x_col.c(), w_col.c()
    _check("qt2_linear_bwd_views", lib().qt2_linear_bwd_views(
        _ptr(dy), M, K, N, seed, ctypes.byref(xc), ctypes.byref(wc), _ptr(dx), _ptr(dw), dw_dtype, _ptr(workspace),
        ws_bytes, _stream(stream)))


def qt2_quant_fwd46_sq_workspace_size(rows: int, cols: int) -> int:
    n = ctypes.c_size_t(0)
    _check("qt2_quant_fwd46_sq_workspace_size", lib().qt2_quant_fwd46_sq_workspace_size(rows, cols, ctypes.byref(n)))
    return n.value


def qt2_quant_fwd46_sq(x: torch.Tensor, rows: int, cols: int, ld: int, row_out: View, col_out: View,
                       workspace: torch.Tensor, ws_bytes: int, stream=None) -> None:
    r, c = row_out.c(), col_out.c()
    _check("qt2_quant_fwd46_sq", lib().qt2_quant_fwd46_sq(_ptr(x), rows, cols, ld, ctypes.byref(r), ctypes.byref(c),
                                                          _ptr(workspace), ws_bytes, _stream(stream)))


def alloc_view_local(R: int, C: int, device="cuda") -> View:
    """A view whose tensor scale is one float per 128 rows (CTA-local quantizer output)."""
    v = alloc_view(R, C, device)
    return View(v.codes, v.scales, torch.empty(R // 128, dtype=torch.float32, device=v.codes.device))


def qt2_quant_fwd46_local(x: torch.Tensor, rows: int, cols: int, ld: int, row_out: View, stream=None) -> None:
    r = row_out.c()
    _check("qt2_quant_fwd46_local", lib().qt2_quant_fwd46_local(_ptr(x), rows, cols, ld, ctypes.byref(r),
                                                                _stream(stream)))


def qt2_gemm_nvfp4_local(a: View, b: View, M: int, N: int, K: int, alpha: float, c: torch.Tensor, c_dtype: int,
                         ldc: int, stream=None) -> None:
    ac, bc = a.c(), b.c()
    _check("qt2_gemm_nvfp4_local", lib().qt2_gemm_nvfp4_local(ctypes.byref(ac), ctypes.byref(bc), M, N, K, alpha,
                                                              _ptr(c), c_dtype, ldc, _stream(stream)))


class fault_hook:
    """Context manager around qt2_set_fault_hook: `decide(site) -> 0/1/2` is asked before every
    CUDA call the library makes while enqueuing (FAULT_NONE, FAULT_FAIL, FAULT_SKIP); the
    sites seen are recorded in `.sites`.  The hook is removed on exit."""

    def __init__(self, decide):
        self.decide, self.sites = decide, []

        def _hook(site, _user):
            name = site.decode()
            self.sites.append(name)
            return int(self.decide(name))
        self._c = FaultHookC(_hook)   # kept alive while installed

    def __enter__(self):
        lib().qt2_set_fault_hook(self._c, None)
        return self

    def __exit__(self, *exc):
        lib().qt2_set_fault_hook(FaultHookC(), None)
        return False


def qt2_selftest_division(exp_lo: int, exp_hi: int, stream=None) -> tuple[int, int]:
    """(reciprocal, division by 6) mismatches of the kernels' forms against IEEE binary32 over
    every value with biased exponent in [exp_lo, exp_hi] (synchronizes)."""
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    _check("qt2_selftest_division", lib().qt2_selftest_division(exp_lo, exp_hi, cnt.data_ptr(), _stream(stream)))
    r, d = cnt.tolist()
    return int(r), int(d)


def qt2_build_checked() -> bool:
    """True when the loaded library is the checked build (QT2_LIBRARY=checked)."""
    return bool(lib().qt2_build_checked())


def qt2_selftest_bounds(stream=None) -> None:
    """Enqueue the store-check self-test (the checked build records QT2_ERR_BOUNDS)."""
    _check("qt2_selftest_bounds", lib().qt2_selftest_bounds(_stream(stream)))


def qt2_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the device wait self-test (its wait gives up after the library's limit)."""
    _check("qt2_selftest_wait_timeout", lib().qt2_selftest_wait_timeout(_stream(stream)))
