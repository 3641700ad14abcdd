"""Replay: the path is stateless, so a step is a function of its inputs, the seed and the tensor
ids.  Running the same one-pass linear step twice (views of X and W from one read each, the
forward GEMM, the backward from those views) gives the same bits everywhere -- every view, Y,
dX and dW (the GEMMs use no atomics: each output tile is accumulated in one fixed order) --
and a different seed changes the MS-EDEN views and the backward outputs but not the forward."""
import pytest
import torch

from nvfp4_quantized_b200 import qt2, synth

pytestmark = pytest.mark.gpu

M, K, N = 2048, 1536, 2560


def _step(x, w, dy, seed):
    vx, vxc = qt2.alloc_view(M, K), qt2.alloc_view(K, M)
    vw, vwc = qt2.alloc_view(N, K), qt2.alloc_view(K, N)
    wsx = qt2.alloc_workspace(qt2.qt2_quant_fwd46_msedEN_col_workspace_size(M, K))
    wsw = qt2.alloc_workspace(qt2.qt2_quant_fwd46_msedEN_col_workspace_size(N, K))
    wsb = qt2.alloc_workspace(qt2.qt2_linear_bwd_views_workspace_size(M, K, N))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    qt2.qt2_quant_fwd46_msedEN_col(x, M, K, K, seed, qt2.QT2_TID_X_COL, vx, vxc, wsx, wsx.numel())
    qt2.qt2_quant_fwd46_msedEN_col(w, N, K, K, seed, qt2.QT2_TID_W_COL, vw, vwc, wsw, wsw.numel())
    qt2.qt2_gemm_nvfp4(vx, vw, M, N, K, 1.0, y, qt2.QT2_DTYPE_BF16, N)
    qt2.qt2_linear_bwd_views(dy, M, K, N, seed, vxc, vwc, dx, dw, qt2.QT2_DTYPE_F32, wsb, wsb.numel())
    torch.cuda.synchronize()
    assert qt2.qt2_device_status() == 0
    views = [t.clone() for v in (vx, vxc, vw, vwc) for t in (v.codes, v.scales, v.tensor_scale)]
    return views, y, dx, dw


def test_replay_is_bit_identical_and_the_seed_matters():
    x, w, dy = [t.cuda() for t in synth.custom_linear_inputs(M, K, N, seed=5)]
    a = _step(x, w, dy, 77)
    b = _step(x, w, dy, 77)
    for ta, tb in zip(a[0], b[0]):
        assert torch.equal(ta, tb)
    for ta, tb in zip(a[1:], b[1:]):
        assert torch.equal(ta.view(torch.int16) if ta.dtype == torch.bfloat16 else ta.view(torch.int32),
                           tb.view(torch.int16) if tb.dtype == torch.bfloat16 else tb.view(torch.int32))
    c = _step(x, w, dy, 78)
    # forward views and Y do not depend on the seed; the column views and the backward do
    for i in (0, 1, 2, 6, 7, 8):
        assert torch.equal(a[0][i], c[0][i])
    assert torch.equal(a[1].view(torch.int16), c[1].view(torch.int16))
    assert not torch.equal(a[0][3], c[0][3]) and not torch.equal(a[0][9], c[0][9])
    assert not torch.equal(a[2].view(torch.int16), c[2].view(torch.int16))
    assert not torch.equal(a[3].view(torch.int32), c[3].view(torch.int32))
