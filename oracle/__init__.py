"""qt2 CPU oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow restatement of the Quartet II NVFP4 linear layer (forward RTN + 4/6, backward
MS-EDEN, GEMM by dequantization with fp64 accumulation), written in plain C
(``qt2_oracle.c``) and driven from here with numpy.  It is used by the test suite, by the
package's ``smoke()`` check and by the benchmark's CPU-baseline leg; nothing on the product
path imports it.  It shares no code with the CUDA library.

The per-function docstrings cite the passage each step follows; the full list of readings
taken where the pages are silent is in the header of ``qt2_oracle.c``.

Parallelism: the C functions take a row range; ``_rows`` below splits rows across Python
threads (ctypes releases the GIL), which changes no arithmetic -- every row is independent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qt2_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libqt2_oracle.so")
_lock = threading.Lock()
_lib = None

TID_SIGNS = 0


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: IEEE binary32 arithmetic, no FMA contraction."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fexcess-precision=standard", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u8, u16, u32, u64 = ctypes.c_uint8, ctypes.c_uint16, ctypes.c_uint32, ctypes.c_uint64
            i64, f32, f64, vp = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
            sig = {
                "or_version": (ctypes.c_int, []),
                "or_bf16_to_f32": (f32, [u16]),
                "or_e2m1_value": (f32, [u8]),
                "or_e2m1_encode": (u8, [f32]),
                "or_e4m3_value": (f32, [u8]),
                "or_e4m3_rne": (u8, [f32]),
                "or_e4m3_sr": (u8, [f32, u32]),
                "or_philox4x32_10": (None, [vp, vp, vp]),
                "or_philox_word": (u32, [u64, u32, u64]),
                "or_rht_signs": (None, [u64, vp]),
                "or_fwht128": (None, [vp]),
                "or_hadamard128_dense": (None, [vp]),
                "or_tree_sum": (f32, [vp, ctypes.c_int]),
                "or_amax_bf16": (f32, [vp, i64]),
                "or_fwd46_tensor_scale": (f32, [f32]),
                "or_fwd46_rows": (None, [vp, i64, i64, f32, i64, i64, vp, vp, vp, vp, vp]),
                "or_fwd46_sq_blocks": (None, [vp, i64, i64, f32, i64, i64, vp, vp, vp, vp, vp]),
                "or_msedEN_rows_stage1": (None, [vp, i64, i64, vp, i64, i64, vp, vp, vp, vp]),
                "or_msedEN_rotated_stage1": (None, [vp, i64, i64, i64, i64, vp, vp, vp, vp]),
                "or_msedEN_rows_stage1_g16": (None, [vp, i64, i64, vp, i64, i64, vp, vp, vp]),
                "or_msedEN_tensor_scale": (f32, [f32]),
                "or_msedEN_finalize": (None, [vp, i64, i64, f32, u64, u32, i64, i64, vp]),
                "or_dequant": (None, [vp, vp, i64, i64, f32, i64, i64, vp]),
                "or_dequant_row": (None, [vp, vp, i64, i64, f32, i64, vp]),
                "or_unrotate_rows": (None, [vp, i64, i64, vp, i64, i64, vp]),
                "or_gemm_f64": (None, [vp, vp, i64, i64, i64, f64, i64, i64, vp]),
                "or_rotated_amax_rows": (f32, [vp, i64, i64, vp, i64, i64]),
                "or_sr_rows_dequant": (None, [vp, i64, i64, vp, f32, u64, u32, i64, i64, vp]),
                "or_sr_tensor_scale": (f32, [f32]),
                "or_sr_rows": (None, [vp, i64, i64, vp, f32, u64, u32, i64, i64, vp, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    return int(os.environ.get("QT2_ORACLE_THREADS", os.cpu_count() or 1))


def _rows(fn, R: int, min_rows: int = 64):
    """Run fn(r0, r1) over [0, R) split across threads; each row is independent."""
    n = max(1, min(threads(), R // max(1, min_rows)))
    if n == 1:
        fn(0, R)
        return
    step = (R + n - 1) // n
    with ThreadPoolExecutor(n) as ex:
        list(ex.map(lambda r0: fn(r0, min(R, r0 + step)), range(0, R, step)))


def _bf16_bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array (accepts a uint16 array or a torch bf16 tensor).

    The method is defined on real numbers only: a tensor holding inf or NaN (exponent field all
    ones) is refused with ValueError, the counterpart of the library's QT2_ERR_NONFINITE."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        b = np.ascontiguousarray(x)
    else:
        import torch
        assert x.dtype == torch.bfloat16
        b = np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    if np.any((b & 0x7F80) == 0x7F80):
        raise ValueError("input holds inf or NaN: the quantizers are defined on finite values only")
    return b


# --------------------------------------------------------------------------- scalar formats
def e2m1_value(code: int) -> float:
    return lib().or_e2m1_value(code)


def e2m1_encode(q: float) -> int:
    return lib().or_e2m1_encode(q)


def e4m3_value(code: int) -> float:
    return lib().or_e4m3_value(code)


def e4m3_rne(v: float) -> int:
    return lib().or_e4m3_rne(v)


def e4m3_sr(v: float, u: int) -> int:
    return lib().or_e4m3_sr(v, u)


def philox4x32_10(ctr, key):
    c = np.array(ctr, dtype=np.uint32)
    k = np.array(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    lib().or_philox4x32_10(_p(c), _p(k), _p(o))
    return [int(v) for v in o]


def philox_word(seed: int, tid: int, j: int) -> int:
    return lib().or_philox_word(seed, tid, j)


def rht_signs(seed: int) -> np.ndarray:
    s = np.zeros(128, dtype=np.float32)
    lib().or_rht_signs(seed, _p(s))
    return s


def fwht128(y) -> np.ndarray:
    v = np.ascontiguousarray(np.array(y, dtype=np.float32).reshape(128))
    lib().or_fwht128(_p(v))
    return v


def hadamard128() -> np.ndarray:
    H = np.zeros((128, 128), dtype=np.float64)
    lib().or_hadamard128_dense(_p(H))
    return H


def tree_sum(v) -> float:
    a = np.ascontiguousarray(np.array(v, dtype=np.float32))
    return lib().or_tree_sum(_p(a), a.size)


def amax_bf16(x) -> float:
    b = _bf16_bits(x)
    return lib().or_amax_bf16(_p(b), b.size)


# --------------------------------------------------------------------------- views
class View:
    """One quantized NVFP4 view in canonical layout: codes [R][C/2] uint8 (element 2j in the
    low nibble), scales [R][C/16] uint8 (E4M3), tensor scale g (fp32).  Rows R are the
    non-contraction axis, C the grouped (contraction) axis."""

    def __init__(self, codes, scales, g, **extra):
        self.codes, self.scales, self.g = codes, scales, np.float32(g)
        self.__dict__.update(extra)

    @property
    def shape(self):
        return self.codes.shape[0], self.codes.shape[1] * 2

    def row_g(self) -> np.ndarray:
        """The tensor scale of every row: g itself, or for a view with one scale per block of
        `row_block` rows (the CTA-local variant) that block's entry of the array g."""
        R = self.shape[0]
        if np.ndim(self.g) == 0:
            return np.full(R, self.g, np.float32)
        return np.repeat(np.asarray(self.g, np.float32), self.row_block)

    def dequant(self) -> np.ndarray:
        """xhat = val(code) * E4M3(scale) * g (g of the row's block for a CTA-local view), fp64
        (the products of a 2-bit, a 4-bit and a 24-bit significand are exact in any order)."""
        R, C = self.shape
        out = np.empty((R, C), dtype=np.float64)
        if np.ndim(self.g) == 0:
            _rows(lambda r0, r1: lib().or_dequant(_p(self.codes), _p(self.scales), R, C, float(self.g), r0, r1,
                                                  _p(out)), R)
            return out
        _rows(lambda r0, r1: lib().or_dequant(_p(self.codes), _p(self.scales), R, C, 1.0, r0, r1, _p(out)), R)
        return out * self.row_g().astype(np.float64)[:, None]

    def dequant_rows(self, rows) -> np.ndarray:
        """Dequantized rows (fp64) of the given row indices only."""
        R, C = self.shape
        rg = self.row_g()
        out = np.empty((len(rows), C), dtype=np.float64)
        for i, r in enumerate(rows):
            row = np.empty(C, dtype=np.float64)
            lib().or_dequant_row(_p(self.codes), _p(self.scales), R, C, 1.0, int(r), _p(row))
            out[i] = row * float(rg[r])
        return out


def fwd46(x, A: float | None = None) -> View:
    """Forward quantizer (RTN onto E2M1 with the per-group 4/6 grid choice) of a bf16 [R][C]
    matrix grouped along C.  A = max|x| over the tensor (computed here unless given)."""
    b = _bf16_bits(x)
    R, C = b.shape
    if A is None:
        A = amax_bf16(b)
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    choice = np.zeros((R, C // 16), np.uint8)
    e6 = np.zeros((R, C // 16), np.float32)
    e4 = np.zeros((R, C // 16), np.float32)
    _rows(lambda r0, r1: lib().or_fwd46_rows(_p(b), R, C, A, r0, r1, _p(codes), _p(scales), _p(choice),
                                             _p(e6), _p(e4)), R)
    return View(codes, scales, lib().or_fwd46_tensor_scale(A), amax=np.float32(A), choice=choice,
                err6=e6, err4=e4)


def fwd46_local(x, row_block: int = 128) -> View:
    """CTA-local forward quantizer ([FAF] "the speed-up is lost between the matmuls": the
    CTA-local NVFP4 variant keeps the scale dependency inside a thread block -- rows and columns
    get their own corrections, constant during the summation and applied after it -- so no
    block waits for the tensor-wide maximum, at the price of a different numeric contract).
    Per block of `row_block` rows: A_b = max|x| over the block (all columns), then the forward
    quantizer of those rows with g_b = A_b/1792.  The view's g is the array of the g_b."""
    b = _bf16_bits(x)
    R, C = b.shape
    assert R % row_block == 0
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    choice = np.zeros((R, C // 16), np.uint8)
    gs = np.empty(R // row_block, np.float32)
    for blk in range(R // row_block):
        r0, r1 = blk * row_block, (blk + 1) * row_block
        A_b = amax_bf16(b[r0:r1])
        lib().or_fwd46_rows(_p(b), R, C, A_b, r0, r1, _p(codes), _p(scales), _p(choice), None, None)
        gs[blk] = lib().or_fwd46_tensor_scale(A_b)
    return View(codes, scales, gs, row_block=row_block, choice=choice)


def transpose_codes(codes: np.ndarray) -> np.ndarray:
    """Packed E2M1 codes of the transposed matrix: [R][C/2] -> [C][R/2] (data movement only)."""
    R, C2 = codes.shape
    nib = np.empty((R, 2 * C2), np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    t = np.ascontiguousarray(nib.T)
    return (t[:, 0::2] | (t[:, 1::2] << 4)).astype(np.uint8)


def fwd46_sq(x, A: float | None = None) -> tuple[View, View]:
    """Square-block forward quantizer of a bf16 [R][C] matrix: one scale per 16x16 block, the
    forward quantizer's RTN and 4/6 choice per block (see or_fwd46_sq_blocks).  Returns the row
    view ([R][C], groups along C) and the column view ([C][R], groups along R): the same
    quantized values, transposed -- the one quantization serves both views of a weight."""
    b = _bf16_bits(x)
    R, C = b.shape
    if A is None:
        A = amax_bf16(b)
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    choice = np.zeros((R // 16, C // 16), np.uint8)
    e6 = np.zeros((R // 16, C // 16), np.float32)
    e4 = np.zeros((R // 16, C // 16), np.float32)
    _rows(lambda b0, b1: lib().or_fwd46_sq_blocks(_p(b), R, C, A, b0, b1, _p(codes), _p(scales), _p(choice),
                                                  _p(e6), _p(e4)), R // 16)
    g = lib().or_fwd46_tensor_scale(A)
    blk = scales[0::16]                                   # [R/16][C/16]: the block scales
    col_scales = np.ascontiguousarray(np.repeat(blk.T, 16, axis=0))   # [C][R/16]
    row = View(codes, scales, g, amax=np.float32(A), choice=choice, err6=e6, err4=e4)
    col = View(transpose_codes(codes), col_scales, g, amax=np.float32(A))
    return row, col


def msedEN(x, seed: int, tid: int, view: str = "row") -> View:
    """MS-EDEN quantizer of a bf16 [R][C] matrix.  view="row": groups along C (the matrix as
    given); view="col": groups along R, i.e. the row view of the transpose [C][R]."""
    b = _bf16_bits(x)
    if view == "col":
        b = np.ascontiguousarray(b.T)
    elif view != "row":
        raise ValueError(view)
    R, C = b.shape
    sgn = rht_signs(seed)
    codes = np.zeros((R, C // 2), np.uint8)
    amax_g = np.zeros((R, C // 16), np.float32)
    P = np.zeros((R, C // 16), np.float32)
    S = np.zeros((R, C // 128), np.float32)
    _rows(lambda r0, r1: lib().or_msedEN_rows_stage1(_p(b), R, C, _p(sgn), r0, r1, _p(codes), _p(amax_g),
                                                     _p(P), _p(S)), R)
    A = float(amax_g.max()) if amax_g.size else 0.0
    if not np.isfinite(A):
        raise ValueError("the rotated values overflow binary32 (|x| above about 2^121)")
    g = lib().or_msedEN_tensor_scale(A)
    scales = np.zeros((R, C // 16), np.uint8)
    _rows(lambda r0, r1: lib().or_msedEN_finalize(_p(P), R, C, g, seed, tid, r0, r1, _p(scales)), R)
    return View(codes, scales, g, amax=np.float32(A), P=P, S=S, amax_g=amax_g, signs=sgn)


def msedEN_group16(x, seed: int, tid: int) -> View:
    """Row view of MS-EDEN with the EDEN factor taken per 16-element group instead of per
    128-element rotation block: the other reading of the grouping the pages leave open, kept to
    compare the two (bias and error); the method itself is msedEN."""
    b = _bf16_bits(x)
    R, C = b.shape
    sgn = rht_signs(seed)
    codes = np.zeros((R, C // 2), np.uint8)
    amax_g = np.zeros((R, C // 16), np.float32)
    P = np.zeros((R, C // 16), np.float32)
    _rows(lambda r0, r1: lib().or_msedEN_rows_stage1_g16(_p(b), R, C, _p(sgn), r0, r1, _p(codes), _p(amax_g),
                                                         _p(P)), R)
    A = float(amax_g.max()) if amax_g.size else 0.0
    if not np.isfinite(A):
        raise ValueError("the rotated values overflow binary32 (|x| above about 2^121)")
    g = lib().or_msedEN_tensor_scale(A)
    scales = np.zeros((R, C // 16), np.uint8)
    _rows(lambda r0, r1: lib().or_msedEN_finalize(_p(P), R, C, g, seed, tid, r0, r1, _p(scales)), R)
    return View(codes, scales, g, amax=np.float32(A), P=P, amax_g=amax_g, signs=sgn)


def msedEN_rows(x, rows, seed: int, tid: int, view: str = "row") -> View:
    """Selected view rows of msedEN(x, seed, tid, view), for views too large to quantize whole
    on the host: the view max A (every rotated value of the whole view, hence its tensor scale g)
    is taken over all rows, then the MS-EDEN steps run on the selected rows only, each row's
    scale draws keyed by its own view-row index as in the whole view.  Returns a View of
    len(rows) rows (codes, scales, the whole view's g, and P, S, amax_g of those rows)."""
    b = _bf16_bits(x)
    if view == "col":
        b = np.ascontiguousarray(b.T)
    elif view != "row":
        raise ValueError(view)
    R, C = b.shape
    sgn = rht_signs(seed)
    A = float(rotated_amax(b, sgn))
    if not np.isfinite(A):
        raise ValueError("the rotated values overflow binary32 (|x| above about 2^121)")
    g = lib().or_msedEN_tensor_scale(A)
    rows = [int(r) for r in rows]
    # whole-view buffers (zero pages; only the selected rows are touched)
    codes = np.zeros((R, C // 2), np.uint8)
    amax_g = np.zeros((R, C // 16), np.float32)
    P = np.zeros((R, C // 16), np.float32)
    S = np.zeros((R, C // 128), np.float32)
    scales = np.zeros((R, C // 16), np.uint8)
    for r in rows:
        lib().or_msedEN_rows_stage1(_p(b), R, C, _p(sgn), r, r + 1, _p(codes), _p(amax_g), _p(P), _p(S))
        lib().or_msedEN_finalize(_p(P), R, C, g, seed, tid, r, r + 1, _p(scales))
    return View(codes[rows], scales[rows], g, amax=np.float32(A), P=P[rows], S=S[rows], amax_g=amax_g[rows])


def msedEN_rotated(y: np.ndarray, seed: int, tid: int) -> View:
    """The MS-EDEN steps on values that are already rotated (fp32 [R][C], C a multiple of 128),
    e.g. by a uniformly random orthogonal map instead of the randomized Hadamard: group scales,
    RTN codes, the EDEN factor per 128-block, the view's tensor scale and the stochastically
    rounded E4M3 scales -- everything msedEN does after its rotation."""
    yf = np.ascontiguousarray(y, dtype=np.float32)
    R, C = yf.shape
    codes = np.zeros((R, C // 2), np.uint8)
    amax_g = np.zeros((R, C // 16), np.float32)
    P = np.zeros((R, C // 16), np.float32)
    S = np.zeros((R, C // 128), np.float32)
    _rows(lambda r0, r1: lib().or_msedEN_rotated_stage1(_p(yf), R, C, r0, r1, _p(codes), _p(amax_g), _p(P), _p(S)),
          R)
    A = float(amax_g.max()) if amax_g.size else 0.0
    if not np.isfinite(A):
        raise ValueError("non-finite rotated values")
    g = lib().or_msedEN_tensor_scale(A)
    scales = np.zeros((R, C // 16), np.uint8)
    _rows(lambda r0, r1: lib().or_msedEN_finalize(_p(P), R, C, g, seed, tid, r0, r1, _p(scales)), R)
    return View(codes, scales, g, amax=np.float32(A), P=P, S=S, amax_g=amax_g)


def unrotate(y: np.ndarray, seed: int) -> np.ndarray:
    """Inverse rotation x = (1/128) D H y per 128-block along the last axis (fp64)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    R, C = y.shape
    out = np.empty_like(y)
    sgn = rht_signs(seed)
    _rows(lambda r0, r1: lib().or_unrotate_rows(_p(y), R, C, _p(sgn), r0, r1, _p(out)), R, min_rows=8)
    return out


def sr_dequant(x, seed: int, tid: int, view: str = "row") -> np.ndarray:
    """Rotated-domain dequantized output of the plain-NVFP4 elementwise-SR baseline."""
    b = _bf16_bits(x)
    if view == "col":
        b = np.ascontiguousarray(b.T)
    R, C = b.shape
    sgn = rht_signs(seed)
    A = lib().or_rotated_amax_rows(_p(b), R, C, _p(sgn), 0, R)
    out = np.zeros((R, C), np.float64)
    _rows(lambda r0, r1: lib().or_sr_rows_dequant(_p(b), R, C, _p(sgn), A, seed, tid, r0, r1, _p(out)), R)
    return out


def rotated_amax(b: np.ndarray, sgn: np.ndarray) -> np.float32:
    """max |y| over a rotated view given as bf16 bits [R][C] (threads over row ranges; max is exact)."""
    R, C = b.shape
    parts = []
    _rows(lambda r0, r1: parts.append(lib().or_rotated_amax_rows(_p(b), R, C, _p(sgn), r0, r1)), R)
    return np.float32(max(parts))


def sr(x, seed: int, tid: int, view: str = "row") -> View:
    """Elementwise-SR NVFP4 view of the rotated tensor, every decision in binary32 (the GPU
    SR baseline's contract): codes, canonical scales and the tensor scale g = A/2688."""
    b = _bf16_bits(x)
    if view == "col":
        b = np.ascontiguousarray(b.T)
    R, C = b.shape
    sgn = rht_signs(seed)
    A = rotated_amax(b, sgn)
    if not np.isfinite(A):
        raise ValueError("the rotated values overflow binary32 (|x| above about 2^121)")
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    _rows(lambda r0, r1: lib().or_sr_rows(_p(b), R, C, _p(sgn), A, seed, tid, r0, r1, _p(codes), _p(scales)), R)
    return View(codes, scales, np.float32(lib().or_sr_tensor_scale(A)))


def gemm(a: np.ndarray, b: np.ndarray, alpha: float = 1.0) -> np.ndarray:
    """C = alpha * A . B^T in fp64 with both operands K-major ([M][K], [N][K])."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    M, K = a.shape
    N = b.shape[0]
    out = np.empty((M, N), np.float64)
    _rows(lambda r0, r1: lib().or_gemm_f64(_p(a), _p(b), M, N, K, alpha, r0, r1, _p(out)), M, min_rows=4)
    return out


def gemm_views(va: View, vb: View, alpha: float = 1.0, rows=None) -> np.ndarray:
    """GEMM of two quantized views by dequantization with fp64 accumulation:
    C = alpha * xhat_A . xhat_B^T (alpha = 2^-7 for MS-EDEN operands, whose rotations cancel
    up to the factor 128).  rows: optional index array of output rows to compute."""
    A = va.dequant()
    B = vb.dequant()
    if rows is not None:
        A = A[np.asarray(rows)]
    return gemm(A, B, alpha)


# Tensor ids of one backward call: 0 = rotation signs, then the four MS-EDEN views.
TID_DY_ROW, TID_DY_COL, TID_W_COL, TID_X_COL = 1, 2, 3, 4


def linear_fwd(x, w):
    """Y = X W^T with both operands quantized by the forward quantizer (fp64 result)."""
    vx, vw = fwd46(x), fwd46(w)
    return gemm_views(vx, vw, 1.0), vx, vw


def linear_bwd(dy, x, w, seed: int):
    """dX = dY W and dW = dY^T X with MS-EDEN operands rotated along the contraction axis
    (fp64 results)."""
    v_dy_row = msedEN(dy, seed, TID_DY_ROW, "row")
    v_w_col = msedEN(w, seed, TID_W_COL, "col")
    v_dy_col = msedEN(dy, seed, TID_DY_COL, "col")
    v_x_col = msedEN(x, seed, TID_X_COL, "col")
    dx = gemm_views(v_dy_row, v_w_col, 2.0 ** -7)
    dw = gemm_views(v_dy_col, v_x_col, 2.0 ** -7)
    return dx, dw, dict(dy_row=v_dy_row, w_col=v_w_col, dy_col=v_dy_col, x_col=v_x_col)
