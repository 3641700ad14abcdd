"""GPU parity of the one-read producer of a layer input's two views (qt2_quant_fwd46_msedEN_col)
and of the backward from pre-quantized column views (qt2_linear_bwd_views), through the C ABI,
against the oracle: the forward view is bit-identical to oracle.fwd46, the column view to
oracle.msedEN(..., "col"), and dX / dW meet the same bars as qt2_linear_bwd's parity tests."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from nvfp4_quantized_b200 import synth
from tests.layout import scales_to_canonical
from tests.test_gpu_linear import _bound_check, _rel
from tests.test_gpu_quant import _assert_view_equal, _inputs

pytestmark = pytest.mark.gpu


def gpu_fused(x: torch.Tensor, seed: int, tid: int, ld_pad: int = 0):
    R, C = x.shape
    if ld_pad:
        big = torch.zeros((R, C + ld_pad), dtype=torch.bfloat16)
        big[:, :C] = x
        xd, ld = big.cuda(), C + ld_pad
    else:
        xd, ld = x.cuda(), C
    vr, vc = qt2.alloc_view(R, C), qt2.alloc_view(C, R)
    ws = qt2.alloc_workspace(qt2.qt2_quant_fwd46_msedEN_col_workspace_size(R, C))
    qt2.qt2_quant_fwd46_msedEN_col(xd, R, C, ld, seed, tid, vr, vc, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    return vr, vc


def _host(v: qt2.View, R: int, C: int):
    return (v.codes.cpu().numpy(), scales_to_canonical(v.scales.cpu().numpy(), R, C),
            np.float32(v.tensor_scale.item()))


# one tile, several tiles each way, non-square, a tall matrix (more tiles than SMs' first wave)
SHAPES = [(128, 128), (256, 384), (384, 640), (1024, 512), (4096, 256)]


@pytest.mark.parametrize("R,C", SHAPES)
@pytest.mark.parametrize("kind", ["gauss", "t3", "zeros"])
def test_fused_views_match_oracle(R, C, kind):
    x = _inputs(kind, R, C, seed=R + C)
    seed, tid = 77 + R, qt2.QT2_TID_X_COL
    vr, vc = gpu_fused(x, seed, tid)
    _assert_view_equal(_host(vr, R, C), O.fwd46(x), "forward view")
    _assert_view_equal(_host(vc, C, R), O.msedEN(x, seed, tid, "col"), "column view")


def test_fused_views_strided_input():
    R, C = 256, 512
    x = _inputs("t3", R, C, seed=5)
    vr, vc = gpu_fused(x, 9, 4, ld_pad=64)
    _assert_view_equal(_host(vr, R, C), O.fwd46(x), "forward view")
    _assert_view_equal(_host(vc, C, R), O.msedEN(x, 9, 4, "col"), "column view")


@pytest.mark.parametrize("shape,seed", [((256, 256, 256), 0), ((384, 640, 1152), 1), ((512, 384, 256), 2)])
def test_linear_bwd_views_matches_oracle(shape, seed):
    M, K, N = shape
    if shape == (256, 256, 256):
        x, w, dy = synth.linear_inputs("tiny", seed)
    else:
        x, w, dy = synth.custom_linear_inputs(M, K, N, seed)
    s = 1234 + seed
    _, x_col = gpu_fused(x, s, qt2.QT2_TID_X_COL)
    w_col = qt2.alloc_view(K, N)
    wsw = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(N, K, qt2.QT2_LAYOUT_COL))
    wd = w.cuda()
    qt2.qt2_quant_msedEN(wd, N, K, K, qt2.QT2_LAYOUT_COL, s, 0, qt2.QT2_TID_W_COL, None, w_col, wsw, wsw.numel())
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ws = qt2.alloc_workspace(qt2.qt2_linear_bwd_views_workspace_size(M, K, N))
    dx_ref, dw_ref, views = O.linear_bwd(dy, x, w, s)
    # the same W view serves two micro-batches: the second run must give the same results
    for _ in range(2):
        qt2.qt2_linear_bwd_views(dy.cuda(), M, K, N, s, x_col, w_col, dx, dw, qt2.QT2_DTYPE_F32, ws, ws.numel())
        assert qt2.qt2_device_status() == 0
        dx_g = dx.float().cpu().numpy().astype(np.float64)
        assert _rel(dx_g, dx_ref) < 4e-3
        _bound_check(dx_g, dx_ref,
                     O.gemm(np.abs(views["dy_row"].dequant()), np.abs(views["w_col"].dequant()), 2 ** -7), True)
        dw_g = dw.cpu().numpy().astype(np.float64)
        assert _rel(dw_g, dw_ref) < 1e-5
        _bound_check(dw_g, dw_ref,
                     O.gemm(np.abs(views["dy_col"].dequant()), np.abs(views["x_col"].dequant()), 2 ** -7), False)


def test_fused_views_full_size():
    """16384 x 8192 layer input with outlier channels (8192 tiles, ~55 per persistent CTA): the
    forward view and the MS-EDEN column view from one read, bit-exact with the oracle."""
    x = synth.make_x(16384, 8192, "t3_outlier_channels", 9)
    seed, tid = 4242, qt2.QT2_TID_X_COL
    vr, vc = gpu_fused(x, seed, tid)
    _assert_view_equal(_host(vr, 16384, 8192), O.fwd46(x), "full-size forward view")
    del vr
    _assert_view_equal(_host(vc, 8192, 16384), O.msedEN(x, seed, tid, "col"), "full-size column view")
