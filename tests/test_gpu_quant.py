"""GPU parity of the quantizers: the CUDA producers (through the C ABI) against the oracle,
bit-exact on packed codes, canonical E4M3 scales and the fp32 tensor scale."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from nvfp4_quantized_b200 import synth
from tests.layout import scales_to_canonical

pytestmark = pytest.mark.gpu


def _bf16(a) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def gpu_fwd46(x: torch.Tensor, ld_pad: int = 0):
    R, C = x.shape
    if ld_pad:
        big = torch.zeros((R, C + ld_pad), dtype=torch.bfloat16)
        big[:, :C] = x
        xd = big.cuda()
        ld = C + ld_pad
    else:
        xd = x.cuda()
        ld = C
    v = qt2.alloc_view(R, C)
    ws = qt2.alloc_workspace(qt2.qt2_quant_fwd46_workspace_size(R, C))
    qt2.qt2_quant_fwd46(xd, R, C, ld, qt2.QT2_LAYOUT_ROW, v, None, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    return (v.codes.cpu().numpy(), scales_to_canonical(v.scales.cpu().numpy(), R, C),
            np.float32(v.tensor_scale.item()))


def gpu_msed(x: torch.Tensor, seed: int, tid_row: int, tid_col: int, mask: int, ld_pad: int = 0):
    R, C = x.shape
    if ld_pad:
        big = torch.zeros((R, C + ld_pad), dtype=torch.bfloat16)
        big[:, :C] = x
        xd, ld = big.cuda(), C + ld_pad
    else:
        xd, ld = x.cuda(), C
    vr = qt2.alloc_view(R, C) if mask & 1 else None
    vc = qt2.alloc_view(C, R) if mask & 2 else None
    ws = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(R, C, mask))
    qt2.qt2_quant_msedEN(xd, R, C, ld, mask, seed, tid_row, tid_col, vr, vc, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    out = {}
    if vr is not None:
        out["row"] = (vr.codes.cpu().numpy(), scales_to_canonical(vr.scales.cpu().numpy(), R, C),
                      np.float32(vr.tensor_scale.item()))
    if vc is not None:
        out["col"] = (vc.codes.cpu().numpy(), scales_to_canonical(vc.scales.cpu().numpy(), C, R),
                      np.float32(vc.tensor_scale.item()))
    return out


def _assert_view_equal(got, ref: O.View, what=""):
    codes, scales, g = got
    assert g == ref.g, (what, g, ref.g)
    bad = np.argwhere(scales != ref.scales)
    assert bad.size == 0, (what, "scales differ at", bad[:5], scales[tuple(bad[0])], ref.scales[tuple(bad[0])])
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, (what, "codes differ at", bad[:5], codes[tuple(bad[0])], ref.codes[tuple(bad[0])])


def _inputs(kind: str, R: int, C: int, seed: int = 0) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    if kind == "gauss":
        return torch.randn((R, C), generator=g).to(torch.bfloat16)
    if kind == "t3":
        return synth.make_x(R, C, "t3_outlier_channels", seed)
    if kind == "lognormal":
        return synth.make_dy(R, C, "lognormal_rows", seed)
    if kind == "weights":
        return synth.make_w(R, C, seed)
    if kind == "zeros":
        return torch.zeros((R, C), dtype=torch.bfloat16)
    if kind == "signed_zeros":
        x = torch.zeros((R, C), dtype=torch.bfloat16)
        x[::2] = -0.0
        x[5, 7] = 3.0
        return x
    if kind == "tiny":
        return (torch.randn((R, C), generator=g) * 1e-34).to(torch.bfloat16)
    if kind == "wide_range":
        x = torch.randn((R, C), generator=g) * torch.exp(torch.randn((R, 1), generator=g) * 6)
        x[:, ::37] *= 1e-6
        return x.to(torch.bfloat16)
    if kind == "exact_grid":
        mags4 = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])
        v = mags4[torch.randint(0, 7, (R, C), generator=g)] * (torch.randint(0, 2, (R, C), generator=g) * 2 - 1)
        v[:, ::16] = 4.0
        return (v * (1792.0 * 2 ** -12 / 4)).to(torch.bfloat16)
    raise ValueError(kind)


FWD_CASES = [((128, 128), "gauss"), ((256, 256), "gauss"), ((384, 640), "t3"), ((256, 1152), "weights"),
             ((128, 256), "zeros"), ((128, 256), "signed_zeros"), ((256, 128), "tiny"), ((256, 512), "wide_range"),
             ((128, 512), "exact_grid"), ((640, 384), "lognormal")]


@pytest.mark.parametrize("shape,kind", FWD_CASES)
def test_fwd46_bitexact(shape, kind):
    x = _inputs(kind, *shape)
    ref = O.fwd46(x)
    _assert_view_equal(gpu_fwd46(x), ref, kind)


def test_fwd46_strided_input():
    x = _inputs("t3", 256, 384, 3)
    _assert_view_equal(gpu_fwd46(x, ld_pad=64), O.fwd46(x), "ld")


MSED_CASES = [((128, 128), "gauss", 0), ((256, 256), "lognormal", 1), ((384, 640), "t3", 2),
              ((256, 1152), "weights", 3), ((128, 256), "zeros", 4), ((256, 128), "tiny", 5),
              ((256, 512), "wide_range", 6), ((640, 384), "gauss", 0xFFFFFFFF12345678)]


@pytest.mark.parametrize("shape,kind,seed", MSED_CASES)
@pytest.mark.parametrize("mask", [qt2.QT2_LAYOUT_ROW, qt2.QT2_LAYOUT_COL, qt2.QT2_LAYOUT_BOTH])
def test_msedEN_bitexact(shape, kind, seed, mask):
    x = _inputs(kind, *shape, seed=seed & 0xFFFF)
    got = gpu_msed(x, seed, 11, 12, mask)
    if mask & 1:
        _assert_view_equal(got["row"], O.msedEN(x, seed, 11, "row"), f"{kind} row")
    if mask & 2:
        _assert_view_equal(got["col"], O.msedEN(x, seed, 12, "col"), f"{kind} col")


def test_msedEN_strided_input():
    x = _inputs("lognormal", 256, 384, 9)
    got = gpu_msed(x, 77, 1, 2, qt2.QT2_LAYOUT_BOTH, ld_pad=128)
    _assert_view_equal(got["row"], O.msedEN(x, 77, 1, "row"), "row ld")
    _assert_view_equal(got["col"], O.msedEN(x, 77, 2, "col"), "col ld")


def test_msedEN_seed_changes_everything_random():
    x = _inputs("gauss", 256, 256, 1)
    a = gpu_msed(x, 1, 1, 2, qt2.QT2_LAYOUT_ROW)["row"]
    b = gpu_msed(x, 2, 1, 2, qt2.QT2_LAYOUT_ROW)["row"]
    assert (a[0] != b[0]).mean() > 0.5          # a new rotation changes most code bytes
    c = gpu_msed(x, 1, 3, 2, qt2.QT2_LAYOUT_ROW)["row"]
    assert np.array_equal(a[0], c[0]) and (a[1] != c[1]).any()   # tensor id only moves the scale draws
