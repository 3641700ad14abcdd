"""GPU parity of the CTA-local forward quantizer and GEMM (qt2_quant_fwd46_local,
qt2_gemm_nvfp4_local, through the C ABI) against the oracle: codes, canonical scales and every
block's tensor scale bit-identical; the GEMM within the GEMM bars."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from tests.layout import scales_to_canonical
from tests.test_gpu_gemm import check as gemm_check
from tests.test_gpu_quant import _inputs

pytestmark = pytest.mark.gpu


def gpu_local(x: torch.Tensor, ld_pad: int = 0) -> qt2.View:
    R, C = x.shape
    if ld_pad:
        big = torch.zeros((R, C + ld_pad), dtype=torch.bfloat16)
        big[:, :C] = x
        xd, ld = big.cuda(), C + ld_pad
    else:
        xd, ld = x.cuda(), C
    v = qt2.alloc_view_local(R, C)
    qt2.qt2_quant_fwd46_local(xd, R, C, ld, v)
    assert qt2.qt2_device_status() == 0
    return v


def _assert_local_equal(v: qt2.View, ref: O.View, R: int, C: int):
    g = v.tensor_scale.cpu().numpy()
    assert np.array_equal(g, ref.g), (g[:4], ref.g[:4])
    assert np.array_equal(scales_to_canonical(v.scales.cpu().numpy(), R, C), ref.scales)
    assert np.array_equal(v.codes.cpu().numpy(), ref.codes)


SHAPES = [(128, 128), (384, 256), (1024, 640), (4096, 2048)]


@pytest.mark.parametrize("R,C", SHAPES)
@pytest.mark.parametrize("kind", ["gauss", "t3", "lognormal", "zeros"])
def test_local_quantizer_matches_oracle(R, C, kind):
    x = _inputs(kind, R, C, seed=R + 7 * C)
    if kind == "gauss" and R >= 384:
        x[128:256] = (x[128:256].float() * 1e-4).to(torch.bfloat16)   # block maxima far apart
    _assert_local_equal(gpu_local(x), O.fwd46_local(x), R, C)


def test_local_quantizer_strided_input():
    R, C = 256, 384
    x = _inputs("t3", R, C, seed=2)
    _assert_local_equal(gpu_local(x, ld_pad=24), O.fwd46_local(x), R, C)


# pair kernel (M, N multiples of 256) and the one-SM kernel (N = 384: 128-wide tiles; M = 384)
@pytest.mark.parametrize("M,N,K", [(512, 768, 1024), (384, 384, 640), (1024, 256, 2048)])
@pytest.mark.parametrize("dtype", [qt2.QT2_DTYPE_F32, qt2.QT2_DTYPE_BF16])
def test_local_gemm_matches_oracle(M, N, K, dtype):
    x = _inputs("lognormal", M, K, seed=3)
    w = _inputs("weights", N, K, seed=4)
    va, vb = gpu_local(x), gpu_local(w)
    ra, rb = O.fwd46_local(x), O.fwd46_local(w)
    out = torch.empty((M, N), dtype=torch.float32 if dtype == qt2.QT2_DTYPE_F32 else torch.bfloat16, device="cuda")
    qt2.qt2_gemm_nvfp4_local(va, vb, M, N, K, 1.0, out, dtype, N)
    assert qt2.qt2_device_status() == 0
    gemm_check(out.float().cpu().numpy().astype(np.float64), ra, rb, 1.0, bf16=dtype == qt2.QT2_DTYPE_BF16)
