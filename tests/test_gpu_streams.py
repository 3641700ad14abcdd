"""Two CUDA streams driving the library at once: each stream quantizes its own tensors (the
forward quantizer's cooperative launch, both views of X from one read, MS-EDEN of dY with both
views) and runs a GEMM on its own views, with no synchronisation between the streams.  Every
view must equal the oracle's bit for bit and every GEMM must meet the GEMM bar, and the device
status word must stay clear: the kernels share no state between calls (each call's scratch is
its own workspace) and the persistent and cooperative launches make progress side by side."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2, synth
from tests.layout import scales_to_canonical

pytestmark = pytest.mark.gpu

R, C, N = 1024, 2048, 768


def _host_view(v, rows, cols):
    return (v.codes.cpu().numpy(), scales_to_canonical(v.scales.cpu().numpy(), rows, cols),
            np.float32(v.tensor_scale.item()))


def _eq(got, ref, what):
    codes, scales, g = got
    assert np.array_equal(codes, ref.codes), what + " codes"
    assert np.array_equal(scales, ref.scales), what + " scales"
    assert g == np.float32(ref.g), what + " tensor scale"


class Job:
    """One stream's work: its inputs, views, workspaces and outputs."""

    def __init__(self, k):
        self.x = synth.make_x(R, C, "t3_outlier_channels", 100 + k)
        self.w = synth.make_w(N, C, 200 + k)
        self.dy = synth.make_dy(R, N, "lognormal_rows", 300 + k)
        self.xd, self.wd, self.dyd = self.x.cuda(), self.w.cuda(), self.dy.cuda()
        self.seed = 0x5151 + k
        self.stream = torch.cuda.Stream()
        self.vx46 = qt2.alloc_view(R, C)
        self.vw46 = qt2.alloc_view(N, C)
        self.vxr, self.vxc = qt2.alloc_view(R, C), qt2.alloc_view(C, R)
        self.vdr, self.vdc = qt2.alloc_view(R, N), qt2.alloc_view(N, R)
        self.ws46 = qt2.alloc_workspace(qt2.qt2_quant_fwd46_workspace_size(R, C))
        self.ws46w = qt2.alloc_workspace(qt2.qt2_quant_fwd46_workspace_size(N, C))
        self.wsf = qt2.alloc_workspace(qt2.qt2_quant_fwd46_msedEN_col_workspace_size(R, C))
        self.wsd = qt2.alloc_workspace(qt2.qt2_quant_msedEN_workspace_size(R, N, qt2.QT2_LAYOUT_BOTH))
        self.y = torch.empty((R, N), dtype=torch.float32, device="cuda")

    def enqueue(self):
        s = self.stream.cuda_stream
        qt2.qt2_quant_fwd46(self.xd, R, C, C, qt2.QT2_LAYOUT_ROW, self.vx46, None, self.ws46, self.ws46.numel(), s)
        qt2.qt2_quant_fwd46(self.wd, N, C, C, qt2.QT2_LAYOUT_ROW, self.vw46, None, self.ws46w, self.ws46w.numel(), s)
        qt2.qt2_quant_fwd46_msedEN_col(self.xd, R, C, C, self.seed, qt2.QT2_TID_X_COL, self.vxr, self.vxc, self.wsf,
                                       self.wsf.numel(), s)
        qt2.qt2_quant_msedEN(self.dyd, R, N, N, qt2.QT2_LAYOUT_BOTH, self.seed, qt2.QT2_TID_DY_ROW,
                             qt2.QT2_TID_DY_COL, self.vdr, self.vdc, self.wsd, self.wsd.numel(), s)
        qt2.qt2_gemm_nvfp4(self.vx46, self.vw46, R, N, C, 1.0, self.y, qt2.QT2_DTYPE_F32, N, s)


def test_two_streams_at_once_match_the_oracle():
    jobs = [Job(0), Job(1)]
    torch.cuda.synchronize()
    for _ in range(3):   # interleave the two streams' launches, several rounds, no syncs between
        for j in jobs:
            j.enqueue()
    torch.cuda.synchronize()
    assert qt2.qt2_device_status() == 0
    for k, j in enumerate(jobs):
        rx = O.fwd46(j.x)
        _eq(_host_view(j.vx46, R, C), rx, f"stream {k} fwd46(X)")
        rw = O.fwd46(j.w)
        _eq(_host_view(j.vw46, N, C), rw, f"stream {k} fwd46(W)")
        _eq(_host_view(j.vxr, R, C), rx, f"stream {k} fused forward view")
        _eq(_host_view(j.vxc, C, R), O.msedEN(j.x, j.seed, qt2.QT2_TID_X_COL, "col"), f"stream {k} fused column view")
        _eq(_host_view(j.vdr, R, N), O.msedEN(j.dy, j.seed, qt2.QT2_TID_DY_ROW, "row"), f"stream {k} dY row")
        _eq(_host_view(j.vdc, N, R), O.msedEN(j.dy, j.seed, qt2.QT2_TID_DY_COL, "col"), f"stream {k} dY col")
        ref = O.gemm_views(rx, rw)
        got = j.y.cpu().numpy().astype(np.float64)
        assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref), f"stream {k} GEMM"
