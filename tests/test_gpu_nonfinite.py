"""Non-finite inputs on the GPU: every quantizer reports inf or NaN in its input (and the
rotating ones an overflowing rotation) as QT2_ERR_NONFINITE through the device status word,
the oracle refuses the same inputs (tests/test_oracle_formats.py), and the next finite call on
the same context is bit-exact again."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from tests.layout import scales_to_canonical

pytestmark = pytest.mark.gpu

R, C = 256, 384


def _bad(value, where=(37, 201)):
    g = torch.Generator().manual_seed(3)
    x = torch.randn((R, C), generator=g).to(torch.bfloat16)
    x[where] = value
    return x.cuda()


def _run_all(xd):
    """Every quantizer entry point on xd; returns the device status after each."""
    out = {}
    ws = qt2.alloc_workspace(1 << 22)
    v, vc = qt2.alloc_view(R, C), qt2.alloc_view(C, R)
    qt2.qt2_quant_fwd46(xd, R, C, C, qt2.QT2_LAYOUT_ROW, v, None, ws, ws.numel())
    out["fwd46"] = qt2.qt2_device_status()
    for mask in (qt2.QT2_LAYOUT_ROW, qt2.QT2_LAYOUT_COL, qt2.QT2_LAYOUT_BOTH):
        qt2.qt2_quant_msedEN(xd, R, C, C, mask, 5, 1, 2, v if mask & 1 else None, vc if mask & 2 else None, ws,
                             ws.numel())
        out[f"msedEN{mask}"] = qt2.qt2_device_status()
        qt2.qt2_quant_sr(xd, R, C, C, mask, 5, 1, 2, v if mask & 1 else None, vc if mask & 2 else None, ws,
                         ws.numel())
        out[f"sr{mask}"] = qt2.qt2_device_status()
    qt2.qt2_quant_fwd46_msedEN_col(xd, R, C, C, 5, 4, v, vc, ws, ws.numel())
    out["fused"] = qt2.qt2_device_status()
    qt2.qt2_quant_fwd46_sq(xd, R, C, C, v, vc, ws, ws.numel())
    out["sq"] = qt2.qt2_device_status()
    vl = qt2.alloc_view_local(R, C)
    qt2.qt2_quant_fwd46_local(xd, R, C, C, vl)
    out["local"] = qt2.qt2_device_status()
    return out


@pytest.mark.parametrize("value", [float("inf"), float("-inf"), float("nan")])
def test_every_quantizer_reports_nonfinite_input(value):
    st = _run_all(_bad(value))
    assert all(s == qt2.QT2_ERR_NONFINITE for s in st.values()), st


def test_rotation_overflow_is_reported_by_the_rotating_quantizers():
    xd = torch.full((R, C), 2.0 ** 125, dtype=torch.bfloat16, device="cuda")
    st = _run_all(xd)
    for k, s in st.items():
        expect = qt2.QT2_ERR_NONFINITE if k.startswith(("msedEN", "sr", "fused")) else 0
        assert s == expect, (k, s)


def test_finite_call_after_a_nonfinite_one_is_exact():
    _run_all(_bad(float("nan")))
    g = torch.Generator().manual_seed(4)
    x = torch.randn((R, C), generator=g).to(torch.bfloat16)
    st = _run_all(x.cuda())
    assert all(s == 0 for s in st.values()), st
    v = qt2.alloc_view(R, C)
    ws = qt2.alloc_workspace(1 << 16)
    qt2.qt2_quant_fwd46(x.cuda(), R, C, C, qt2.QT2_LAYOUT_ROW, v, None, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    ref = O.fwd46(x)
    assert np.array_equal(v.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(scales_to_canonical(v.scales.cpu().numpy(), R, C), ref.scales)
