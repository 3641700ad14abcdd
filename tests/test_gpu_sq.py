"""GPU parity of the square-block forward quantizer (qt2_quant_fwd46_sq, through the C ABI)
against the oracle: both views bit-identical (codes, canonical scales, tensor scale), and both
views usable as GEMM operands (fp32 output within the GEMM bars)."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from tests.layout import scales_to_canonical
from tests.test_gpu_gemm import check as gemm_check
from tests.test_gpu_quant import _assert_view_equal, _inputs

pytestmark = pytest.mark.gpu


def gpu_sq(x: torch.Tensor, ld_pad: int = 0):
    R, C = x.shape
    if ld_pad:
        big = torch.zeros((R, C + ld_pad), dtype=torch.bfloat16)
        big[:, :C] = x
        xd, ld = big.cuda(), C + ld_pad
    else:
        xd, ld = x.cuda(), C
    vr, vc = qt2.alloc_view(R, C), qt2.alloc_view(C, R)
    ws = qt2.alloc_workspace(qt2.qt2_quant_fwd46_sq_workspace_size(R, C))
    qt2.qt2_quant_fwd46_sq(xd, R, C, ld, vr, vc, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    return vr, vc


def _host(v: qt2.View, R: int, C: int):
    return (v.codes.cpu().numpy(), scales_to_canonical(v.scales.cpu().numpy(), R, C),
            np.float32(v.tensor_scale.item()))


# one tile; several each way; non-square; the 1.9B-class layer's W [8192][2048] in full
SHAPES = [(128, 128), (256, 384), (640, 384), (2048, 1024), (8192, 2048)]


@pytest.mark.parametrize("R,C", SHAPES)
@pytest.mark.parametrize("kind", ["weights", "gauss", "t3", "zeros"])
def test_sq_views_match_oracle(R, C, kind):
    if (R, C) == (8192, 2048) and kind != "weights":
        pytest.skip("full size runs on the weight distribution only")
    x = _inputs(kind, R, C, seed=R * 3 + C)
    vr, vc = gpu_sq(x)
    ref_r, ref_c = O.fwd46_sq(x)
    _assert_view_equal(_host(vr, R, C), ref_r, "row view")
    _assert_view_equal(_host(vc, C, R), ref_c, "column view")


def test_sq_strided_input():
    R, C = 256, 512
    x = _inputs("t3", R, C, seed=11)
    vr, vc = gpu_sq(x, ld_pad=40)
    ref_r, ref_c = O.fwd46_sq(x)
    _assert_view_equal(_host(vr, R, C), ref_r, "row view")
    _assert_view_equal(_host(vc, C, R), ref_c, "column view")


def _upload(v: O.View) -> qt2.View:
    from tests.layout import canonical_to_scales
    return qt2.View(torch.from_numpy(v.codes).cuda(), torch.from_numpy(canonical_to_scales(v.scales)).cuda(),
                    torch.tensor([float(v.g)], dtype=torch.float32).cuda())


def test_sq_views_as_gemm_operands():
    """Y = X W^T with W's row view and dX = dY W with W's column view (unrotated operands)."""
    M, K, N = 512, 768, 256
    w = _inputs("weights", N, K, seed=3)
    x = _inputs("gauss", M, K, seed=4)
    dy = _inputs("gauss", M, N, seed=5)
    vr, vc = gpu_sq(w)
    ref_r, ref_c = O.fwd46_sq(w)
    vx, vdy = O.fwd46(x), O.fwd46(dy)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    qt2.qt2_gemm_nvfp4(_upload(vx), vr, M, N, K, 1.0, y, qt2.QT2_DTYPE_F32, N)
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    qt2.qt2_gemm_nvfp4(_upload(vdy), vc, M, K, N, 1.0, dx, qt2.QT2_DTYPE_F32, K)
    assert qt2.qt2_device_status() == 0
    gemm_check(y.cpu().numpy().astype(np.float64), vx, ref_r, 1.0)
    gemm_check(dx.cpu().numpy().astype(np.float64), vdy, ref_c, 1.0)
