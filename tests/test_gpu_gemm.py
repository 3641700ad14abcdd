"""GPU parity of the block-scaled NVFP4 GEMM: the tcgen05 kernel (through the C ABI) consumes
views produced by the oracle and is compared with the oracle's fp64 product of the dequantized
operands.  Bar (fp32 output): relative Frobenius error <= 1e-5 and, elementwise,
|err| <= 1e-4 * sum_k |a_ik| |b_jk|.  bf16 output adds its own rounding (2^-9 relative)."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from tests.layout import canonical_to_scales

pytestmark = pytest.mark.gpu


def upload(view: O.View) -> qt2.View:
    return qt2.View(torch.from_numpy(view.codes).cuda(), torch.from_numpy(canonical_to_scales(view.scales)).cuda(),
                    torch.tensor([float(view.g)], dtype=torch.float32).cuda())


def gpu_gemm(va: O.View, vb: O.View, alpha: float, dtype: int):
    M, K = va.shape
    N = vb.shape[0]
    out = torch.empty((M, N), dtype=torch.float32 if dtype == qt2.QT2_DTYPE_F32 else torch.bfloat16, device="cuda")
    a, b = upload(va), upload(vb)
    qt2.qt2_gemm_nvfp4(a, b, M, N, K, alpha, out, dtype, N)
    assert qt2.qt2_device_status() == 0
    return out.float().cpu().numpy().astype(np.float64)


def check(got, va, vb, alpha, bf16=False):
    A, B = va.dequant(), vb.dequant()
    ref = O.gemm(A, B, alpha)
    bound = O.gemm(np.abs(A), np.abs(B), abs(alpha))
    err = np.abs(got - ref)
    if bf16:
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-4 * bound + 1e-30)
        assert np.linalg.norm(got - ref) <= 4e-3 * np.linalg.norm(ref) + 1e-30
    else:
        assert np.all(err <= 1e-4 * bound + 1e-30), np.max(err / (bound + 1e-30))
        assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref) + 1e-30, \
            np.linalg.norm(got - ref) / np.linalg.norm(ref)


def _x(R, C, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((R, C), generator=g) * scale).to(torch.bfloat16)


# (M, N, K): single tile, N % 256 != 0 (128-wide tiles), K not a multiple of 256 (half stage),
# several stages around the ring, a long K.
SHAPES = [(128, 128, 128), (128, 256, 256), (256, 256, 256), (384, 640, 1152), (256, 512, 2048), (128, 384, 4224),
          (256, 256, 8192),
          # M and N multiples of 256 run on SM pairs: several tiles each way, a K tail (4224 = 16.5 x 256),
          # and more tiles (16 x 16) than resident pairs, so each pair loops over tiles; M < N with
          # more tiles than pairs (the tile order that runs along M first)
          (512, 768, 1024), (768, 512, 4224), (4096, 4096, 512), (1024, 9728, 768)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("dtype", [qt2.QT2_DTYPE_F32, qt2.QT2_DTYPE_BF16])
def test_gemm_forward_operands(M, N, K, dtype):
    va = O.fwd46(_x(M, K, 1))
    vb = O.fwd46(_x(N, K, 2, 0.02))
    got = gpu_gemm(va, vb, 1.0, dtype)
    check(got, va, vb, 1.0, bf16=dtype == qt2.QT2_DTYPE_BF16)


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (384, 640, 1152), (128, 384, 4224), (512, 1024, 2048)])
def test_gemm_msedEN_operands(M, N, K):
    seed = 5
    va = O.msedEN(_x(M, K, 3, 1e-4), seed, 1, "row")
    vb = O.msedEN(_x(N, K, 4, 0.02), seed, 3, "row")
    got = gpu_gemm(va, vb, 2.0 ** -7, qt2.QT2_DTYPE_F32)
    check(got, va, vb, 2.0 ** -7)


def test_gemm_zero_and_extreme_scales():
    M = N = K = 256
    x = _x(M, K, 6)
    x[:128] = 0.0
    va = O.fwd46(x)
    vb = O.fwd46(_x(N, K, 7) * 3e4)
    got = gpu_gemm(va, vb, 1.0, qt2.QT2_DTYPE_F32)
    assert np.all(got[:128] == 0.0)
    check(got, va, vb, 1.0)


# Output with a leading dimension larger than N, and a base 16 bytes off a 32-byte boundary: the
# pair kernel stores 32 bytes at a time only when every row start is 32-byte aligned, else 16.
# (dtype, extra columns, start offset in elements)
PADDED = [(qt2.QT2_DTYPE_BF16, 8, 0), (qt2.QT2_DTYPE_BF16, 16, 0), (qt2.QT2_DTYPE_F32, 8, 4),
          (qt2.QT2_DTYPE_F32, 8, 0)]


@pytest.mark.parametrize("dtype,pad,off", PADDED)
def test_gemm_strided_output(dtype, pad, off):
    M, N, K = 512, 768, 1024
    va = O.fwd46(_x(M, K, 8))
    vb = O.fwd46(_x(N, K, 9, 0.02))
    tdt = torch.float32 if dtype == qt2.QT2_DTYPE_F32 else torch.bfloat16
    ldc = N + pad
    buf = torch.full((off + M * ldc + 64,), 7.0, dtype=tdt, device="cuda")
    out = buf[off:off + M * ldc].view(M, ldc)
    qt2.qt2_gemm_nvfp4(upload(va), upload(vb), M, N, K, 1.0, out, dtype, ldc)
    assert qt2.qt2_device_status() == 0
    got = out[:, :N].float().cpu().numpy().astype(np.float64)
    check(got, va, vb, 1.0, bf16=dtype == qt2.QT2_DTYPE_BF16)
    assert torch.all(out[:, N:] == 7.0)          # padding columns untouched
    assert torch.all(buf[:off] == 7.0) and torch.all(buf[off + M * ldc:] == 7.0)
