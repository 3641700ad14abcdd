"""Parity at the largest point of the quantizer sweep: 2^30 elements as 262144 rows of 4096
(bf16 N(0,1) with 0.1% of the elements x50, the sweep's own input), in the launch
configuration the sweep times.  The oracle cannot quantize the whole tensor in a test's time,
so the tensor-wide quantities it needs are taken over every element (the forward quantizer's
max |x|, each MS-EDEN view's max |y| over every rotated block) and sampled rows of every view
-- the first and last rows, rows at tile and wave boundaries, random rows -- are compared with
the oracle byte for byte: codes, scales and the tensor scale."""
import numpy as np
import pytest

import oracle as O
from nvfp4_quantized_b200 import qt2, synth
from tests.layout import scale_rows_to_canonical

pytestmark = pytest.mark.gpu

L = 4096
R = synth.sweep_rows(30, L)


def _sample(n_rows, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 255, 256, n_rows // 2, n_rows - 129, n_rows - 128, n_rows - 1]
    return sorted(set(fixed) | set(int(r) for r in rng.integers(0, n_rows, 22)))


@pytest.fixture(scope="module")
def tensors():
    assert R * L == 1 << 30
    xd = synth.sweep_tensor(30, L, seed=30, device="cuda")
    return xd, xd.cpu()


def _rows_of(view, rows, n_rows, n_cols):
    codes = view.codes.cpu().numpy()[rows]
    scales = scale_rows_to_canonical(view.scales.cpu().numpy(), rows, n_cols)
    return codes, scales, np.float32(view.tensor_scale.item())


def test_forward_quantizer_at_2_30(tensors):
    xd, x = tensors
    v = qt2.alloc_view(R, L)
    ws = qt2.alloc_workspace(qt2.qt2_quant_fwd46_workspace_size(R, L))
    qt2.qt2_quant_fwd46(xd, R, L, L, qt2.QT2_LAYOUT_ROW, v, None, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    A = O.amax_bf16(x)
    rows = _sample(R, 1)
    ref = O.fwd46(x[rows], A=A)
    codes, scales, g = _rows_of(v, rows, R, L)
    assert g == ref.g
    assert np.array_equal(codes, ref.codes)
    assert np.array_equal(scales, ref.scales)


def test_msedEN_both_views_at_2_30(tensors):
    xd, x = tensors
    seed = 0x2030
    vr, vc = qt2.alloc_view(R, L), qt2.alloc_view(L, R)
    ws = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(R, L, qt2.QT2_LAYOUT_BOTH))
    qt2.qt2_quant_msedEN(xd, R, L, L, qt2.QT2_LAYOUT_BOTH, seed, 1, 2, vr, vc, ws, ws.numel())
    assert qt2.qt2_device_status() == 0
    rows = _sample(R, 2)
    ref = O.msedEN_rows(x, rows, seed, 1, "row")
    codes, scales, g = _rows_of(vr, rows, R, L)
    assert g == ref.g
    assert np.array_equal(codes, ref.codes)
    assert np.array_equal(scales, ref.scales)
    cols = _sample(L, 3)
    refc = O.msedEN_rows(x, cols, seed, 2, "col")
    codes, scales, g = _rows_of(vc, cols, L, R)
    assert g == refc.g
    assert np.array_equal(codes, refc.codes)
    assert np.array_equal(scales, refc.scales)
