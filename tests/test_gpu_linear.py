"""GPU parity of the composed linear layer (qt2_linear_fwd / qt2_linear_bwd through the C ABI)
against the oracle's fp64 results on the same seeded inputs.

Small cases compare every output; the full-size cases (the 1.9B-class layer: tokens 16384,
d_in 2048, d_out 8192; the Llama-3-8B MLP gate/up 4096 -> 14336 and down 14336 -> 4096 linears
at 16384 tokens, the launch configurations the benchmark times) compare every quantized view
bit for bit with the oracle, and the GEMM outputs on sampled rows the oracle computes one by
one from those views."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from nvfp4_quantized_b200 import synth
from tests.layout import scales_to_canonical
from tests.test_gpu_quant import _assert_view_equal

pytestmark = pytest.mark.gpu


def run_linear(x, w, dy, seed, dw_dtype=qt2.QT2_DTYPE_F32):
    M, K = x.shape
    N = w.shape[0]
    xd, wd, dyd = x.cuda(), w.cuda(), dy.cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32 if dw_dtype == qt2.QT2_DTYPE_F32 else torch.bfloat16, device="cuda")
    wsf = qt2.alloc_workspace(qt2.qt2_linear_fwd_workspace_size(M, K, N))
    wsb = qt2.alloc_workspace(qt2.qt2_linear_bwd_workspace_size(M, K, N))
    qt2.qt2_linear_fwd(xd, wd, M, K, N, y, wsf, wsf.numel())
    qt2.qt2_linear_bwd(dyd, xd, wd, M, K, N, seed, dx, dw, dw_dtype, wsb, wsb.numel())
    assert qt2.qt2_device_status() == 0
    return y, dx, dw


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _bound_check(got, ref, bound, bf16):
    err = np.abs(got - ref)
    tol = 1e-4 * bound + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0) + 1e-30
    assert np.all(err <= tol), np.max(err / tol)


@pytest.mark.parametrize("shape,seed", [((256, 256, 256), 0), ((384, 640, 1152), 1), ((512, 384, 256), 2)])
def test_linear_matches_oracle(shape, seed):
    M, K, N = shape
    if shape == (256, 256, 256):
        x, w, dy = synth.linear_inputs("tiny", seed)
    else:
        x, w, dy = synth.custom_linear_inputs(M, K, N, seed)
    y, dx, dw = run_linear(x, w, dy, seed=1234 + seed)
    y_ref, vx, vw = O.linear_fwd(x, w)
    dx_ref, dw_ref, views = O.linear_bwd(dy, x, w, 1234 + seed)

    y_g = y.float().cpu().numpy().astype(np.float64)
    assert _rel(y_g, y_ref) < 4e-3
    _bound_check(y_g, y_ref, O.gemm(np.abs(vx.dequant()), np.abs(vw.dequant())), True)

    dx_g = dx.float().cpu().numpy().astype(np.float64)
    assert _rel(dx_g, dx_ref) < 4e-3
    _bound_check(dx_g, dx_ref, O.gemm(np.abs(views["dy_row"].dequant()), np.abs(views["w_col"].dequant()), 2 ** -7),
                 True)

    dw_g = dw.cpu().numpy().astype(np.float64)
    assert _rel(dw_g, dw_ref) < 1e-5
    _bound_check(dw_g, dw_ref, O.gemm(np.abs(views["dy_col"].dequant()), np.abs(views["x_col"].dequant()), 2 ** -7),
                 False)


def test_linear_bwd_bf16_dw():
    x, w, dy = synth.linear_inputs("tiny", 3)
    _, _, dw = run_linear(x, w, dy, seed=9, dw_dtype=qt2.QT2_DTYPE_BF16)
    _, dw_ref, _ = O.linear_bwd(dy, x, w, 9)
    assert _rel(dw.float().cpu().numpy().astype(np.float64), dw_ref) < 4e-3


def _full_view(view: qt2.View, R, C):
    return (view.codes.cpu().numpy(), scales_to_canonical(view.scales.cpu().numpy(), R, C),
            np.float32(view.tensor_scale.item()))


@pytest.mark.parametrize("config", ["llm1p9b", "mlp8b_up", "mlp8b_down", "stack1p1b_qkv", "stack1p1b_down"])
def test_full_size_views_and_layer(config):
    """Full-size layer in the launch configuration the benchmark times: EVERY code, scale and
    tensor scale of every quantized view (forward views of X and W, MS-EDEN views of dY both
    ways, W's and X's column views) equals the oracle's; Y, dX and dW of the layer call match
    the oracle's fp64 products of those views on sampled rows.  At these sizes every
    persistent producer wraps its tile ring many times per CTA and the forward quantizer's
    grid-stride loop covers millions of groups per launch."""
    M, K, N = synth.SHAPES[config]
    x, w, dy = synth.linear_inputs(config, 0)
    seed = 2024
    y, dx, dw = run_linear(x, w, dy, seed)
    xd, wd, dyd = x.cuda(), w.cuda(), dy.cuda()
    rng = np.random.default_rng(0)
    rows_m = np.sort(rng.choice(M, 6, replace=False))
    rows_n = np.sort(rng.choice(N, 6, replace=False))

    # forward views, full tensors (the calls qt2_linear_fwd makes)
    def fwd_view(t, R, C):
        v = qt2.alloc_view(R, C)
        ws = qt2.alloc_workspace(qt2.qt2_quant_fwd46_workspace_size(R, C))
        qt2.qt2_quant_fwd46(t, R, C, C, qt2.QT2_LAYOUT_ROW, v, None, ws, ws.numel())
        assert qt2.qt2_device_status() == 0
        return _full_view(v, R, C)

    o_x = O.fwd46(x)
    _assert_view_equal(fwd_view(xd, M, K), o_x, f"{config} fwd46 X")
    o_w = O.fwd46(w)
    _assert_view_equal(fwd_view(wd, N, K), o_w, f"{config} fwd46 W")
    y_ref = O.gemm(o_x.dequant_rows(rows_m), o_w.dequant(), 1.0)
    y_g = y[torch.from_numpy(rows_m).cuda()].float().cpu().numpy().astype(np.float64)
    assert _rel(y_g, y_ref) < 4e-3
    _bound_check(y_g, y_ref, O.gemm(np.abs(o_x.dequant_rows(rows_m)), np.abs(o_w.dequant()), 1.0), True)
    del o_x, o_w

    # MS-EDEN views, full tensors (the calls qt2_linear_bwd makes)
    def msed_views(t, R, C, mask, tid_row, tid_col):
        vr = qt2.alloc_view(R, C) if mask & 1 else None
        vc = qt2.alloc_view(C, R) if mask & 2 else None
        ws = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(R, C, mask))
        qt2.qt2_quant_msedEN(t, R, C, C, mask, seed, tid_row, tid_col, vr, vc, ws, ws.numel())
        assert qt2.qt2_device_status() == 0
        return (_full_view(vr, R, C) if vr is not None else None, _full_view(vc, C, R) if vc is not None else None)

    g_dy_row, g_dy_col = msed_views(dyd, M, N, qt2.QT2_LAYOUT_BOTH, qt2.QT2_TID_DY_ROW, qt2.QT2_TID_DY_COL)
    o_dy_row = O.msedEN(dy, seed, qt2.QT2_TID_DY_ROW, "row")
    _assert_view_equal(g_dy_row, o_dy_row, f"{config} MS-EDEN dY row")
    del g_dy_row
    _, g_w_col = msed_views(wd, N, K, qt2.QT2_LAYOUT_COL, 0, qt2.QT2_TID_W_COL)
    o_w_col = O.msedEN(w, seed, qt2.QT2_TID_W_COL, "col")
    _assert_view_equal(g_w_col, o_w_col, f"{config} MS-EDEN W col")
    del g_w_col
    dx_ref = O.gemm(o_dy_row.dequant_rows(rows_m), o_w_col.dequant(), 2.0 ** -7)
    dx_g = dx[torch.from_numpy(rows_m).cuda()].float().cpu().numpy().astype(np.float64)
    assert _rel(dx_g, dx_ref) < 4e-3
    _bound_check(dx_g, dx_ref, O.gemm(np.abs(o_dy_row.dequant_rows(rows_m)), np.abs(o_w_col.dequant()), 2.0 ** -7),
                 True)
    del o_dy_row, o_w_col

    o_dy_col = O.msedEN(dy, seed, qt2.QT2_TID_DY_COL, "col")
    _assert_view_equal(g_dy_col, o_dy_col, f"{config} MS-EDEN dY col")
    del g_dy_col
    _, g_x_col = msed_views(xd, M, K, qt2.QT2_LAYOUT_COL, 0, qt2.QT2_TID_X_COL)
    o_x_col = O.msedEN(x, seed, qt2.QT2_TID_X_COL, "col")
    _assert_view_equal(g_x_col, o_x_col, f"{config} MS-EDEN X col")
    del g_x_col
    dw_ref = O.gemm(o_dy_col.dequant_rows(rows_n), o_x_col.dequant(), 2.0 ** -7)
    dw_g = dw[torch.from_numpy(rows_n).cuda()].cpu().numpy().astype(np.float64)
    assert _rel(dw_g, dw_ref) < 1e-5
    _bound_check(dw_g, dw_ref, O.gemm(np.abs(o_dy_col.dequant_rows(rows_n)), np.abs(o_x_col.dequant()), 2.0 ** -7),
                 False)
