"""The benchmark's step schedules, checked on the host with a recording stand-in for the
binding (no GPU): every schedule runs the three GEMMs of every linear on the views that belong
to them, each backward GEMM's two operands are quantized with the one seed of that step (the
rotation must cancel in the product), the one-pass schedule quantizes each distinct tensor
once a step, and the timed-call names line up with the calls issued."""
import types

import pytest

import bench
from nvfp4_quantized_b200 import synth


class _View:
    def __init__(self, tag):
        self.tag = tag
        self.made_by = None     # (call, seed) of the quantizer that last wrote it


class FakeQ(types.SimpleNamespace):
    QT2_LAYOUT_ROW, QT2_LAYOUT_COL, QT2_LAYOUT_BOTH = 1, 2, 3
    QT2_DTYPE_BF16, QT2_DTYPE_F32 = 0, 1
    QT2_TID_SIGNS, QT2_TID_DY_ROW, QT2_TID_DY_COL, QT2_TID_W_COL, QT2_TID_X_COL = 0, 1, 2, 3, 4

    def __init__(self):
        super().__init__()
        self.calls = []
        self.n = 0

    # allocation
    def alloc_view(self, r, c, dev=None):
        self.n += 1
        return _View(f"v{self.n}[{r}x{c}]")

    alloc_view_local = alloc_view

    def alloc_workspace(self, n, dev=None):
        return types.SimpleNamespace(numel=lambda: n)

    def __getattr__(self, name):
        if name.endswith("_workspace_size"):
            return lambda *a: 256
        raise AttributeError(name)

    # quantizers: record which tensor went in and stamp the views they write
    def qt2_quant_fwd46(self, x, r, c, ld, mask, row, col, ws, n, st=None):
        self.calls.append(("fwd46", id(x), None))
        row.made_by = ("fwd46", id(x), None)

    def qt2_quant_msedEN(self, x, r, c, ld, mask, seed, tr, tc, row, col, ws, n, st=None):
        self.calls.append(("msedEN", id(x), seed))
        for v in (row, col):
            if v is not None:
                v.made_by = ("msedEN", id(x), seed)

    def qt2_quant_fwd46_msedEN_col(self, x, r, c, ld, seed, tid, row, col, ws, n, st=None):
        self.calls.append(("fused", id(x), seed))
        row.made_by = ("fwd46", id(x), None)
        col.made_by = ("msedEN", id(x), seed)

    def qt2_quant_fwd46_local(self, x, r, c, ld, v, st=None):
        self.calls.append(("fwd46_local", id(x), None))
        v.made_by = ("fwd46_local", id(x), None)

    def qt2_gemm_nvfp4(self, a, b, M, N, K, alpha, c, dt, ldc, st=None):
        self.calls.append(("gemm", a.made_by, b.made_by))

    qt2_gemm_nvfp4_local = qt2_gemm_nvfp4


def _run(config, schedule, steps=2):
    Q = FakeQ()
    linears = synth.stack_linears(config)
    sets = []
    for s in range(2):
        d, seen = {}, {}
        for name, M, K, N, xk, dk, shared in linears:
            x = seen[shared] if shared else object()
            seen[name] = x
            d[name] = (x, object(), object())
        sets.append(d)
    states = {n: bench.LayerState.__new__(bench.LayerState) for n, *_ in linears}
    for (n, M, K, N, *_), stt in zip(linears, states.values()):
        # LayerState's constructor allocates device tensors; build the same fields on the fake
        stt.M, stt.K, stt.N = M, K, N
        stt.y = stt.dx = stt.dw = object()
        stt.vx, stt.vw = Q.alloc_view(M, K), Q.alloc_view(N, K)
        stt.v_dy_row, stt.v_dy_col = Q.alloc_view(M, N), Q.alloc_view(N, M)
        stt.v_w_col, stt.v_x_col = Q.alloc_view(K, N), Q.alloc_view(K, M)
        stt.vxl, stt.vwl = Q.alloc_view(M, K), Q.alloc_view(N, K)
        for w in ("ws46", "ws46b", "ws_dy", "ws_w", "ws_x", "ws_xv", "ws_wv"):
            setattr(stt, w, Q.alloc_workspace(256))
    setup = len(Q.calls)
    step = bench.make_step(Q, linears, sets, states, schedule, None)
    setup = len(Q.calls) - setup
    marks_all = []
    for i in range(steps):
        before = len(Q.calls)
        marks = []
        step(i, lambda j: marks.append((j, len(Q.calls))))
        marks_all.append((before, marks))
    return Q, linears, sets, setup, marks_all


@pytest.mark.parametrize("config", ["mlp8b", "stack1p1b", "llm1p9b"])
@pytest.mark.parametrize("schedule", ["onepass", "separate", "fused", "local"])
def test_gemm_operands_and_shared_rotation(config, schedule):
    Q, linears, sets, setup, marks_all = _run(config, schedule)
    names = bench.call_names(linears, schedule)
    for i, (before, marks) in enumerate(marks_all):
        # one mark before every timed call and one after the last; each timed call is one call
        assert [j for j, _ in marks] == list(range(len(names) + 1))
        pos = [p for _, p in marks]
        assert all(b - a == 1 for a, b in zip(pos, pos[1:]))
        assert pos[0] == before
        calls = Q.calls[before:pos[-1]]
        gemms = [c for c in calls if c[0] == "gemm"]
        assert len(gemms) == 3 * len(linears)
        x_ids = {n: id(sets[i % 2][n][0]) for n, *_ in linears}
        w_ids = {n: id(sets[i % 2][n][1]) for n, *_ in linears}
        dy_ids = {n: id(sets[i % 2][n][2]) for n, *_ in linears}
        for k, (name, *_) in enumerate(linears):
            fwd, dgrad, wgrad = gemms[3 * k:3 * k + 3]
            fw = "fwd46_local" if schedule == "local" else "fwd46"
            assert fwd[1] == (fw, x_ids[name], None)
            if schedule != "fused":   # W's forward view is made before the timed steps there
                assert fwd[2] == (fw, w_ids[name], None)
            # dgrad: dY's row view with W's column view; wgrad: dY's column view with X's
            assert dgrad[1][:2] == ("msedEN", dy_ids[name]) and wgrad[1][:2] == ("msedEN", dy_ids[name])
            assert wgrad[2][:2] == ("msedEN", x_ids[name])
            assert dgrad[2][0] == "msedEN"
            # the rotation is shared: both operands of each backward GEMM carry one seed
            assert dgrad[1][2] == dgrad[2][2] and wgrad[1][2] == wgrad[2][2]
        if schedule != "fused":
            assert w_ids[linears[0][0]] == gemms[0][2][1]


@pytest.mark.parametrize("config", ["mlp8b", "stack1p1b"])
def test_onepass_quantizes_each_tensor_once_per_step_with_a_new_seed(config):
    Q, linears, sets, setup, marks_all = _run(config, "onepass", steps=3)
    assert setup == 0
    seeds = []
    for i, (before, marks) in enumerate(marks_all):
        calls = [c for c in Q.calls[before:marks[-1][1]] if c[0] != "gemm"]
        srcs = [c[1] for c in calls]
        assert len(srcs) == len(set(srcs)), "a tensor was quantized twice in one step"
        distinct_x = {id(sets[i % 2][n][0]) for n, *_ in linears}
        assert len(calls) == len(distinct_x) + 2 * len(linears)   # X views, W views, dY views
        assert {c[2] for c in calls} == {calls[0][2]}               # one seed for the whole step
        seeds.append(calls[0][2])
    assert len(set(seeds)) == len(seeds)


def test_clock_reasons_that_force_a_second_measurement():
    """The sampler's summary names the NVML clock-event reasons seen under load; hardware and
    thermal slowdowns make the bench measure again, the power cap alone does not."""
    c = bench.ClockSampler(0)
    c.max_mhz = 1965
    c.samples = [(1965, 600.0, 0x4), (1965, 620.0, 0x4), (1200, 10.0, 0x8)]   # the idle sample is ignored
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert not set(s["reasons"]) & bench.THROTTLE_REASONS
    c.samples = [(1965, 600.0, 0x4), (1700, 640.0, 0x4 | 0x40)]
    s = c.summary()
    assert set(s["reasons"]) == {"sw_power_cap", "hw_thermal_slowdown"}
    assert set(s["reasons"]) & bench.THROTTLE_REASONS
