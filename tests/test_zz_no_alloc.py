"""The workspace-free MS-EDEN entry point, qt2_quant_msedEN_noalloc.

It exists for callers that cannot give the library device memory for scratch (for example a
runtime that has split all device memory among its own pools, or a latency-critical path that
must not call cudaMalloc): its scratch lives in a fixed array inside the library instead.  Its
results must be exactly those of qt2_quant_msedEN, call after call, although every call reuses
the same array -- so each call is compared with the workspace entry point, several calls in a
row, with inputs chosen so that leftovers of an earlier call (a larger view maximum, different
pre-scales) would show up as wrong scales.
"""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_quantized_b200 import qt2


def _noalloc(x, rows, cols, mask, seed, tid_row, tid_col):
    """Call the C entry point directly through the C ABI."""
    vr = qt2.alloc_view(rows, cols) if mask & 1 else None
    vc = qt2.alloc_view(cols, rows) if mask & 2 else None
    r = vr.c() if vr is not None else None
    c = vc.c() if vc is not None else None
    st = qt2.lib().qt2_quant_msedEN_noalloc(x.data_ptr(), rows, cols, cols, mask, seed, tid_row, tid_col,
                                            ctypes.byref(r) if r else None, ctypes.byref(c) if c else None,
                                            torch.cuda.current_stream().cuda_stream)
    assert st == qt2.QT2_OK, qt2.status_string(st)
    return vr, vc


def _with_workspace(x, rows, cols, mask, seed, tid_row, tid_col):
    vr = qt2.alloc_view(rows, cols) if mask & 1 else None
    vc = qt2.alloc_view(cols, rows) if mask & 2 else None
    ws = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(rows, cols, mask))
    qt2.qt2_quant_msedEN(x, rows, cols, cols, mask, seed, tid_row, tid_col, vr, vc, ws, ws.numel())
    return vr, vc


def _same(a: qt2.View, b: qt2.View):
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert torch.equal(a.tensor_scale, b.tensor_scale)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    g = torch.Generator().manual_seed(42)
    calls = [
        # (rows, cols, mask, seed, input scale): a large-magnitude tensor first, then smaller
        # ones, so a view maximum left over from an earlier call would change the scales
        (512, 1024, qt2.QT2_LAYOUT_BOTH, 11, 1e3),
        (256, 384, qt2.QT2_LAYOUT_BOTH, 12, 1e-4),
        (384, 256, qt2.QT2_LAYOUT_ROW, 13, 1.0),
        (256, 640, qt2.QT2_LAYOUT_COL, 14, 3e-2),
    ]
    for rows, cols, mask, seed, scale in calls:
        x = (torch.randn((rows, cols), generator=g) * scale).to(torch.bfloat16).cuda()
        got_r, got_c = _noalloc(x, rows, cols, mask, seed, 1, 2)
        ref_r, ref_c = _with_workspace(x, rows, cols, mask, seed, 1, 2)
        torch.cuda.synchronize()
        assert qt2.qt2_device_status() == 0
        if mask & 1:
            _same(got_r, ref_r)
        if mask & 2:
            _same(got_c, ref_c)
    # the same call twice in a row gives the same bytes
    x = (torch.randn((256, 256), generator=g)).to(torch.bfloat16).cuda()
    a_r, a_c = _noalloc(x, 256, 256, qt2.QT2_LAYOUT_BOTH, 5, 1, 2)
    b_r, b_c = _noalloc(x, 256, 256, qt2.QT2_LAYOUT_BOTH, 5, 1, 2)
    torch.cuda.synchronize()
    _same(a_r, b_r)
    _same(a_c, b_c)


@pytest.mark.gpu
def test_noalloc_at_the_largest_accepted_size():
    """8192 x 8192 with both views fills the built-in scratch exactly: the results are the
    workspace entry point's, bit for bit, on two calls in a row (the second with a smaller input,
    so a view maximum left over from the first would change its scales)."""
    g = torch.Generator(device="cuda").manual_seed(7)
    for seed, scale in ((21, 1.0), (22, 1e-3)):
        x = (torch.randn((8192, 8192), generator=g, device="cuda") * scale).to(torch.bfloat16)
        got_r, got_c = _noalloc(x, 8192, 8192, qt2.QT2_LAYOUT_BOTH, seed, 1, 2)
        ref_r, ref_c = _with_workspace(x, 8192, 8192, qt2.QT2_LAYOUT_BOTH, seed, 1, 2)
        torch.cuda.synchronize()
        assert qt2.qt2_device_status() == 0
        _same(got_r, ref_r)
        _same(got_c, ref_c)
        del x, got_r, got_c, ref_r, ref_c


def test_noalloc_rejects_tensors_beyond_the_builtin_scratch():
    """A tensor whose scratch would not fit in the built-in array is refused before any work
    (fake, never-dereferenced device addresses: the check runs on the host first)."""
    v = qt2.NVFP4ViewC(0x10000, 0x20000, 0x30000)
    rows, cols = 16384, 8192        # both views need 64 MiB of pre-scales, above the 32 MiB array
    st = qt2.lib().qt2_quant_msedEN_noalloc(0x1000, rows, cols, cols, qt2.QT2_LAYOUT_BOTH, 1, 1, 2,
                                            ctypes.byref(v), ctypes.byref(v), None)
    assert st == qt2.QT2_ERR_WORKSPACE
    assert qt2.qt2_quant_msedEN_workspace_size(rows, cols, qt2.QT2_LAYOUT_BOTH) > 32 * 1024 * 1024
