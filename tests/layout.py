"""Test-side helpers: un-permute the tensor-core scale-factor order of a view's scales into the
canonical [R][C/16] order, following the formula stated in include/qt2.h."""
import numpy as np


def scale_offsets(R: int, C: int) -> np.ndarray:
    """offsets[r, j] = byte offset of the scale of row r, group j."""
    r = np.arange(R)[:, None]
    j = np.arange(C // 16)[None, :]
    return ((r // 128) * (C // 64) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)


def scales_to_canonical(buf: np.ndarray, R: int, C: int) -> np.ndarray:
    return np.asarray(buf).reshape(-1)[scale_offsets(R, C)]


def canonical_to_scales(canon: np.ndarray) -> np.ndarray:
    R, G = canon.shape
    out = np.zeros(R * G, np.uint8)
    out[scale_offsets(R, G * 16)] = canon
    return out


def scale_rows_to_canonical(buf: np.ndarray, rows, C: int) -> np.ndarray:
    """Canonical [len(rows)][C/16] scales of the given rows only (same offsets as scale_offsets)."""
    r = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(C // 16)[None, :]
    off = ((r // 128) * (C // 64) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)
    return np.asarray(buf).reshape(-1)[off]
