"""Benchmark of the Quartet II NVFP4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config mlp8b]
                    [--schedule onepass|separate|fused|local] [--sweep] [--op fwd46_sq]

A step is one pass of the whole hot path over one batch, for every linear layer of the
workload: the forward quantizer on X and W (tensor max + RTN/4-6), the forward GEMM, MS-EDEN on
dY (row and column views in one pass), on W (column view) and on X (column view) with their
scale passes, and the dgrad and wgrad GEMMs, issued one C-ABI call at a time so that each
kernel's duration is taken with CUDA events inside the timed region.

Workloads (nvfp4_quantized_b200.synth, seeded synthetic bf16 tensors):
  mlp8b (default)  the Llama-3-8B MLP at 16384 tokens: gate and up 4096 -> 14336 (one shared
                   X), down 14336 -> 4096; 9 GEMMs, 1.73e13 FLOP a step.
  stack1p1b        the five linears of a 1.1B-class block at 32768 tokens (QKV, O, gate, up,
                   down; d_model 2048, FFN 5632); 15 GEMMs, 1.01e13 FLOP a step.
  llm1p9b          one 1.9B-class linear, 16384 tokens, 2048 -> 8192.
  mlp8b_up, mlp8b_down   one MLP linear each.
Every step's inputs exceed L2 (126 MB) many times over, and two input sets alternate between
steps, so no step starts with its inputs in L2.

Schedules: onepass (default: every tensor of the step quantized once, both of its views from
one read -- X's and W's forward and MS-EDEN column views through qt2_quant_fwd46_msedEN_col, X
once for linears that read the same X, dY's two MS-EDEN views in one pass -- with a new seed
every step, so the step does all of its work); separate (each linear as qt2_linear_fwd/bwd
would run it: one quantizer call per view, X quantized per linear); fused (NEXT-1 with W's two
views made once before the timed steps and one seed, as for the micro-batches of one optimizer
step); local (the forward with CTA-local scales, a different numeric contract).  All but local
produce the same bits for the same seed.

Beside our numbers the line carries: torch bf16 matmuls on the same shapes and GPU (the pages'
speed claims are relative to BF16), `e2e` through qt2_linear_fwd/bwd with every step's
activations and gradients uploaded from pinned host memory and its outputs downloaded (W
resident, as a parameter is), `e2e_resident` (the same API calls on resident tensors), and the
oracle timed on the host cores (`cpu_baseline`, all cores and one thread).

--sweep times both quantizers alone over 2^20..2^30 elements, rows of 2048 / 4096 / 14336,
ROW / COL / BOTH views, L2 flushed between calls.  --op fwd46_sq times the square-block weight
quantizer alone.

Multi-GPU (torchrun, one rank per GPU): the path has no exchange step, so every rank runs the
same step on its own token batch (weak scaling, no collective on the data path); the time is
the max over ranks and value = all ranks' FLOPs / that time.

--impl reference times the CPU oracle (the plain restatement the CUDA path is checked against)
on a bounded sample of the same workload, on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Quartet II linear fwd+bwd TFLOPS; quantizer GB/s; % of FP4/HBM roofline"
UNIT = "TFLOP/s"
FP4_PER_BF16 = 4.0     # nominal dense NVFP4 / BF16 tensor throughput (9 / 2.25 PFLOP/s)

# Algorithmic bytes per input element of each quantizer call (reads + writes the method needs).
BYTES_FWD46 = 2 + 2 + 0.5 + 1 / 16            # max pass read, quantize read, codes, scales
BYTES_MSED_ONE = 2 + 0.5 + 0.25 + 0.25 + 1 / 16  # read, codes, pre-scale write + read, scales
BYTES_MSED_BOTH = 2 + 2 * (0.5 + 0.25 + 0.25 + 1 / 16)
BYTES_FUSED_X = 2 + 2 + (0.5 + 1 / 16) + (0.5 + 0.25 + 0.25 + 1 / 16)   # max read, read, both views
BYTES_FWD46_SQ = 2 + 2 + 2 * (0.5 + 1 / 16)   # max read, read, row and column views


def peaks():
    """Measured HBM copy bandwidth and cuBLAS bf16 throughput of this GPU pool (burst: a kernel
    timed alone; sustained: a seconds-long loop under the power cap), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------------------- clocks
# clock-event reasons that make a timed run invalid (sw_power_cap is kept and reported)
THROTTLE_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    """Samples the SM clock, power and clock-event reasons through NVML every 2 ms while the
    timed region runs (read-only queries; no setting is touched).  NVML is opened and the
    sampling thread started before the warm-up, so the whole timed region is covered; the
    region's first and last samples are taken synchronously by begin() and end()."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        import threading
        self.gpu, self.period = gpu_index, period_s
        self.samples = []
        self.max_mhz, self.error, self._h = None, None, None
        self._ready, self._stop, self._rec = threading.Event(), threading.Event(), threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        import pynvml
        sm = pynvml.nvmlDeviceGetClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        pw = pynvml.nvmlDeviceGetPowerUsage(self._h) / 1000.0
        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        self.samples.append((sm, pw, rs))

    def _run(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # NVML unavailable: report that, never fail the run
            self.error = repr(e)
            self._ready.set()
            return
        self._ready.set()
        while not self._stop.is_set():
            if self._rec.is_set():
                try:
                    self._sample()
                except Exception as e:
                    self.error = repr(e)
            self._stop.wait(self.period)

    def start(self):
        self._t.start()
        return self

    def begin(self):
        self._ready.wait(timeout=30)
        if self._h is not None:
            self._sample()
        self._rec.set()

    def end(self):
        self._rec.clear()
        if self._h is not None:
            self._sample()

    def stop(self):
        self._stop.set()
        self._t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0,
                    "error": self.error}
        loaded = [s for s in self.samples if s[1] > 250.0] or self.samples
        sm = sorted(s[0] for s in loaded)
        reasons = sorted({n for s in loaded for n, bit in self.REASONS.items() if s[2] & bit})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "samples_under_load": len(loaded),
                "power_w_max": max(s[1] for s in self.samples), "source": "nvml, 2 ms period"}


# ---------------------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank passes its own device-timed milliseconds and gets the
    maximum back (one all-reduce; a single rank returns its own)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own batch (weak scaling), so the
    job does world * steps * flops in the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def rank_input_seed(rank: int, set_index: int) -> int:
    """Seed of input set `set_index` (two alternate) on `rank`: each rank draws its own batch."""
    return 1000 * rank + 10 * set_index


# ---------------------------------------------------------------------------------------- step
SCHEDULE_NOTE = {
    "onepass": "per step and linear: X's forward (RTN+4/6) and MS-EDEN column views from one read "
               "(once for linears that read the same X: gate and up), W's two views from one read, the "
               "forward GEMM, MS-EDEN of dY (both views, one read), dgrad and wgrad GEMMs; a new seed every "
               "step",
    "separate": "per step and linear: fwd46(X), fwd46(W), forward GEMM, MS-EDEN of dY (both views), of W "
                "(column view) and of X (column view), dgrad and wgrad GEMMs; a new seed every step",
    "fused": "per step and linear: X's two views from one read (once per shared X), forward GEMM, MS-EDEN of "
             "dY, dgrad and wgrad GEMMs; W's views made once before the timed steps and one seed for all "
             "steps (the micro-batches of one optimizer step)",
    "local": "as separate, with the forward's CTA-local scales (qt2_quant_fwd46_local, qt2_gemm_nvfp4_local)",
}


def step_flops(config: str) -> float:
    from nvfp4_quantized_b200 import synth
    return sum(3 * 2.0 * M * N * K for _, M, K, N, *_ in synth.stack_linears(config))


def call_names(linears, schedule: str):
    """(linear name, call name) of every timed call of one step, in order."""
    out = []
    seen_x = set()
    for name, M, K, N, xk, dk, shared in linears:
        if schedule == "fused":
            calls = ([] if shared in seen_x else ["fused_x_views"]) + ["gemm_fwd", "msed_dy_both", "gemm_dgrad",
                                                                      "gemm_wgrad"]
        elif schedule == "onepass":
            calls = ([] if shared in seen_x else ["fused_x_views"]) + ["fused_w_views", "gemm_fwd", "msed_dy_both",
                                                                      "gemm_dgrad", "gemm_wgrad"]
        elif schedule == "local":
            calls = ["fwd46_local_x", "fwd46_local_w", "gemm_fwd", "msed_dy_both", "msed_w_col", "msed_x_col",
                     "gemm_dgrad", "gemm_wgrad"]
        else:
            calls = ["fwd46_x", "fwd46_w", "gemm_fwd", "msed_dy_both", "msed_w_col", "msed_x_col", "gemm_dgrad",
                     "gemm_wgrad"]
        seen_x.add(name)
        out += [(name, c) for c in calls]
    return out


def call_work(call: str, M: int, K: int, N: int):
    """('gemm', FLOPs) or ('quant', algorithmic bytes) of one call on a linear M x K -> N."""
    if call.startswith("gemm_"):
        return "gemm", 2.0 * M * N * K
    return "quant", {"fwd46_x": M * K * BYTES_FWD46, "fwd46_w": N * K * BYTES_FWD46,
                     "fwd46_local_x": M * K * BYTES_FWD46, "fwd46_local_w": N * K * BYTES_FWD46,
                     "msed_dy_both": M * N * BYTES_MSED_BOTH, "msed_w_col": N * K * BYTES_MSED_ONE,
                     "msed_x_col": M * K * BYTES_MSED_ONE, "fused_x_views": M * K * BYTES_FUSED_X,
                     "fused_w_views": N * K * BYTES_FUSED_X}[call]


class LayerState:
    """Device buffers of one linear: views, outputs and workspaces."""

    def __init__(self, Q, M, K, N, dev, local=False):
        import torch
        self.M, self.K, self.N = M, K, N
        COL, BOTH = Q.QT2_LAYOUT_COL, Q.QT2_LAYOUT_BOTH
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.dw = torch.empty((N, K), dtype=torch.float32, device=dev)
        self.vx, self.vw = Q.alloc_view(M, K, dev), Q.alloc_view(N, K, dev)
        self.v_dy_row, self.v_dy_col = Q.alloc_view(M, N, dev), Q.alloc_view(N, M, dev)
        self.v_w_col, self.v_x_col = Q.alloc_view(K, N, dev), Q.alloc_view(K, M, dev)
        self.ws46 = Q.alloc_workspace(Q.qt2_quant_fwd46_workspace_size(max(M, N), K), dev)
        self.ws46b = Q.alloc_workspace(Q.qt2_quant_fwd46_workspace_size(max(M, N), K), dev)
        self.ws_dy = Q.alloc_workspace(Q.qt2_quant_msedEN_workspace_size(M, N, BOTH), dev)
        self.ws_w = Q.alloc_workspace(Q.qt2_quant_msedEN_workspace_size(N, K, COL), dev)
        self.ws_x = Q.alloc_workspace(Q.qt2_quant_msedEN_workspace_size(M, K, COL), dev)
        self.ws_xv = Q.alloc_workspace(Q.qt2_quant_fwd46_msedEN_col_workspace_size(M, K), dev)
        self.ws_wv = Q.alloc_workspace(Q.qt2_quant_fwd46_msedEN_col_workspace_size(N, K), dev)
        if local:
            self.vxl, self.vwl = Q.alloc_view_local(M, K, dev), Q.alloc_view_local(N, K, dev)


def make_step(Q, linears, sets, states, schedule, stream):
    """step(i, marks) runs one step on input set i % 2; marks(j) is called before call j and once
    after the last call (for the per-call CUDA events)."""
    ROW, COL, BOTH = Q.QT2_LAYOUT_ROW, Q.QT2_LAYOUT_COL, Q.QT2_LAYOUT_BOTH
    seed0 = 0x5EED0000

    if schedule == "fused":
        # W's views, made once for every micro-batch of the optimizer step: the column view (the
        # backward seed of those micro-batches) and the forward view (RTN of an unchanged W)
        for name, M, K, N, *_ in linears:
            st, w = states[name], sets[0][name][1]
            Q.qt2_quant_msedEN(w, N, K, K, COL, seed0, 0, Q.QT2_TID_W_COL, None, st.v_w_col, st.ws_w,
                               st.ws_w.numel(), stream)
            Q.qt2_quant_fwd46(w, N, K, K, ROW, st.vw, None, st.ws46b, st.ws46b.numel(), stream)

    def step(i, mark=lambda j: None):
        seed = seed0 if schedule == "fused" else seed0 + i
        j = 0
        for name, M, K, N, xk, dk, shared in linears:
            x, w, dy = sets[i % 2][name]
            st = states[name]
            if schedule in ("fused", "onepass"):
                if shared is None:
                    mark(j); j += 1
                    Q.qt2_quant_fwd46_msedEN_col(x, M, K, K, seed, Q.QT2_TID_X_COL, st.vx, st.v_x_col, st.ws_xv,
                                                 st.ws_xv.numel(), stream)
                if schedule == "onepass":
                    # W's forward view and MS-EDEN column view from one read, every step
                    mark(j); j += 1
                    Q.qt2_quant_fwd46_msedEN_col(w, N, K, K, seed, Q.QT2_TID_W_COL, st.vw, st.v_w_col, st.ws_wv,
                                                 st.ws_wv.numel(), stream)
                vx, vxc = (states[shared].vx, states[shared].v_x_col) if shared else (st.vx, st.v_x_col)
                mark(j); j += 1
                Q.qt2_gemm_nvfp4(vx, st.vw, M, N, K, 1.0, st.y, Q.QT2_DTYPE_BF16, N, stream)
                mark(j); j += 1
                Q.qt2_quant_msedEN(dy, M, N, N, BOTH, seed, Q.QT2_TID_DY_ROW, Q.QT2_TID_DY_COL, st.v_dy_row,
                                   st.v_dy_col, st.ws_dy, st.ws_dy.numel(), stream)
                mark(j); j += 1
                Q.qt2_gemm_nvfp4(st.v_dy_row, st.v_w_col, M, K, N, 2.0 ** -7, st.dx, Q.QT2_DTYPE_BF16, K, stream)
                mark(j); j += 1
                Q.qt2_gemm_nvfp4(st.v_dy_col, vxc, N, K, M, 2.0 ** -7, st.dw, Q.QT2_DTYPE_F32, K, stream)
                continue
            mark(j); j += 1
            if schedule == "local":
                Q.qt2_quant_fwd46_local(x, M, K, K, st.vxl, stream)
                mark(j); j += 1
                Q.qt2_quant_fwd46_local(w, N, K, K, st.vwl, stream)
                mark(j); j += 1
                Q.qt2_gemm_nvfp4_local(st.vxl, st.vwl, M, N, K, 1.0, st.y, Q.QT2_DTYPE_BF16, N, stream)
            else:
                Q.qt2_quant_fwd46(x, M, K, K, ROW, st.vx, None, st.ws46, st.ws46.numel(), stream)
                mark(j); j += 1
                Q.qt2_quant_fwd46(w, N, K, K, ROW, st.vw, None, st.ws46b, st.ws46b.numel(), stream)
                mark(j); j += 1
                Q.qt2_gemm_nvfp4(st.vx, st.vw, M, N, K, 1.0, st.y, Q.QT2_DTYPE_BF16, N, stream)
            mark(j); j += 1
            Q.qt2_quant_msedEN(dy, M, N, N, BOTH, seed, Q.QT2_TID_DY_ROW, Q.QT2_TID_DY_COL, st.v_dy_row,
                               st.v_dy_col, st.ws_dy, st.ws_dy.numel(), stream)
            mark(j); j += 1
            Q.qt2_quant_msedEN(w, N, K, K, COL, seed, 0, Q.QT2_TID_W_COL, None, st.v_w_col, st.ws_w,
                               st.ws_w.numel(), stream)
            mark(j); j += 1
            Q.qt2_quant_msedEN(x, M, K, K, COL, seed, 0, Q.QT2_TID_X_COL, None, st.v_x_col, st.ws_x,
                               st.ws_x.numel(), stream)
            mark(j); j += 1
            Q.qt2_gemm_nvfp4(st.v_dy_row, st.v_w_col, M, K, N, 2.0 ** -7, st.dx, Q.QT2_DTYPE_BF16, K, stream)
            mark(j); j += 1
            Q.qt2_gemm_nvfp4(st.v_dy_col, st.v_x_col, N, K, M, 2.0 ** -7, st.dw, Q.QT2_DTYPE_F32, K, stream)
        mark(j)

    return step


def torch_bf16_leg(linears, sets, dev, reps: int = 10):
    """torch.matmul in bf16 on the same shapes and GPU: fwd X.W^T, dgrad dY.W, wgrad dY^T.X per
    linear, each timed alone with CUDA events (3 warm-up, `reps` timed, median)."""
    import torch
    out, total = {}, 0.0
    for name, M, K, N, *_ in linears:
        x, w, dy = sets[0][name]
        ops = {"fwd": lambda: torch.matmul(x, w.t()), "dgrad": lambda: torch.matmul(dy, w),
               "wgrad": lambda: torch.matmul(dy.t(), x)}
        per = {}
        for op, fn in ops.items():
            for _ in range(3):
                fn()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            per[op] = sorted(ts)[len(ts) // 2]
        out[name] = {op: {"ms": ms, "tflops": 2.0 * M * N * K / (ms * 1e-3) / 1e12} for op, ms in per.items()}
        total += sum(per.values())
    return {"ms_per_step": total, "per_linear": out, "dtype": "bf16 inputs, fp32 accumulate (cuBLAS via torch)",
            "timing": "each matmul alone, CUDA events, median of 10 after 3 warm-up"}


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from nvfp4_quantized_b200 import qt2 as Q, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    linears = synth.stack_linears(args.config)
    sets = [synth.stack_inputs(args.config, seed=rank_input_seed(rank, i), device=dev) for i in range(2)]
    states = {name: LayerState(Q, M, K, N, dev, local=args.schedule == "local")
              for name, M, K, N, *_ in linears}
    stream = torch.cuda.current_stream(dev)
    names = call_names(linears, args.schedule)
    step = make_step(Q, linears, sets, states, args.schedule, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    clk = ClockSampler(local_rank).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert Q.qt2_device_status(stream) == 0, "device status word set during warm-up"

    def timed(clk, first_step):
        """The timed region: exactly args.steps steps between a barrier + synchronize on each
        side, clocks sampled throughout; returns (elapsed ms, per-call ms, launches, clocks)."""
        events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        # every CUDA call the library makes is announced to the hook: count the kernel launches
        counter = Q.fault_hook(lambda site: Q.FAULT_NONE)
        clk.begin()
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with counter:
            t_start.record(stream)
            for i in range(args.steps):
                ev = events[i]
                step(first_step + i, lambda j, ev=ev: ev[j].record(stream))
            t_end.record(stream)
        torch.cuda.synchronize()
        clk.end()
        clk.stop()
        barrier()
        per = [sum(events[i][j].elapsed_time(events[i][j + 1]) for i in range(args.steps)) / args.steps
               for j in range(len(names))]
        return t_start.elapsed_time(t_end), per, counter.sites.count("launch"), clk.summary()

    elapsed_ms, per, launches, clocks = timed(clk, args.warmup)
    # A run that saw a hardware or thermal slowdown is measured once more (every rank takes the
    # same decision: the flag is the max over ranks); the line reports the second run and says so.
    throttled = 1.0 if set(clocks.get("reasons", [])) & THROTTLE_REASONS else 0.0
    if max_over_ranks(throttled, world, dev) > 0:
        first = {"ms_per_step": elapsed_ms / args.steps, "reasons": clocks.get("reasons")}
        elapsed_ms, per, launches, clocks = timed(ClockSampler(local_rank).start(), args.warmup + args.steps)
        clocks["remeasured_after"] = first
    status = Q.qt2_device_status(stream)
    max_ms = max_over_ranks(elapsed_ms, world, dev)

    torch_leg = None if args.no_torch else torch_bf16_leg(linears, sets, dev)
    e2e = e2e_res = None
    if not args.no_e2e:
        e2e, e2e_res = run_e2e(args, Q, linears, sets, dev, world, barrier)
    return dict(linears=linears, names=names, max_ms=max_ms, per=per, status=status, clocks=clocks,
                e2e=e2e, e2e_resident=e2e_res, torch=torch_leg, launches=launches)


def run_e2e(args, Q, linears, sets, dev, world, barrier):
    """End to end through the public API (qt2_linear_fwd + qt2_linear_bwd per linear).

    `e2e`: every step uploads its activations X and output gradients dY from pinned host memory
    and downloads Y, dX and dW; W is uploaded once and stays resident, as a parameter does.
    Three streams (upload, compute, download) and two device buffer sets pipeline consecutive
    steps, so PCIe runs both ways at once; events order each buffer set's reuse.
    `e2e_resident`: the same API calls on resident device tensors, no copies (the API's own
    overhead over the kernels)."""
    import torch
    hosts, bufs = {}, [{}, {}]
    h2d = d2h = 0
    for name, M, K, N, xk, dk, shared in linears:
        x, w, dy = sets[0][name]
        hx = hosts[shared]["x"] if shared else x.cpu().pin_memory()
        hosts[name] = dict(x=hx, dy=dy.cpu().pin_memory(),
                           y=torch.empty((M, N), dtype=torch.bfloat16).pin_memory(),
                           dx=torch.empty((M, K), dtype=torch.bfloat16).pin_memory(),
                           dw=torch.empty((N, K), dtype=torch.float32).pin_memory())
        h2d += (0 if shared else hx.numel() * 2) + dy.numel() * 2
        d2h += M * N * 2 + M * K * 2 + N * K * 4
        for b in range(2):
            bufs[b][name] = dict(x=bufs[b][shared]["x"] if shared else torch.empty_like(x), w=w,
                                 dy=torch.empty_like(dy), y=torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                                 dx=torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                                 dw=torch.empty((N, K), dtype=torch.float32, device=dev))
    onepass = args.schedule == "onepass"
    if onepass:
        # the public calls of the one-pass schedule: both views of X (once per shared X) and of
        # W from one read each, the forward GEMM, and the backward from those column views
        views = {n: dict(vx=Q.alloc_view(M, K, dev), vxc=Q.alloc_view(K, M, dev), vw=Q.alloc_view(N, K, dev),
                         vwc=Q.alloc_view(K, N, dev),
                         wsx=Q.alloc_workspace(Q.qt2_quant_fwd46_msedEN_col_workspace_size(M, K), dev),
                         wsw=Q.alloc_workspace(Q.qt2_quant_fwd46_msedEN_col_workspace_size(N, K), dev),
                         wsb=Q.alloc_workspace(Q.qt2_linear_bwd_views_workspace_size(M, K, N), dev))
                 for n, M, K, N, *_ in linears}
        api = ("qt2_quant_fwd46_msedEN_col on X (once per shared X) and on W, qt2_gemm_nvfp4, "
               "qt2_linear_bwd_views per linear")
    else:
        wsf = {n: Q.alloc_workspace(Q.qt2_linear_fwd_workspace_size(M, K, N), dev) for n, M, K, N, *_ in linears}
        wsb = {n: Q.alloc_workspace(Q.qt2_linear_bwd_workspace_size(M, K, N), dev) for n, M, K, N, *_ in linears}
        api = "qt2_linear_fwd + qt2_linear_bwd per linear"
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def compute(B, i, cs):
        if onepass:
            seed = 0xE2E0 + i
            for name, M, K, N, xk, dk, shared in linears:
                d, v = B[name], views[name]
                vs = views[shared] if shared else v
                if shared is None:
                    Q.qt2_quant_fwd46_msedEN_col(d["x"], M, K, K, seed, Q.QT2_TID_X_COL, v["vx"], v["vxc"], v["wsx"],
                                                 v["wsx"].numel(), cs)
                Q.qt2_quant_fwd46_msedEN_col(d["w"], N, K, K, seed, Q.QT2_TID_W_COL, v["vw"], v["vwc"], v["wsw"],
                                             v["wsw"].numel(), cs)
                Q.qt2_gemm_nvfp4(vs["vx"], v["vw"], M, N, K, 1.0, d["y"], Q.QT2_DTYPE_BF16, N, cs)
                Q.qt2_linear_bwd_views(d["dy"], M, K, N, seed, vs["vxc"], v["vwc"], d["dx"], d["dw"],
                                       Q.QT2_DTYPE_F32, v["wsb"], v["wsb"].numel(), cs)
            return
        for name, M, K, N, *_ in linears:
            d = B[name]
            Q.qt2_linear_fwd(d["x"], d["w"], M, K, N, d["y"], wsf[name], wsf[name].numel(), cs)
            Q.qt2_linear_bwd(d["dy"], d["x"], d["w"], M, K, N, 0xE2E0 + i, d["dx"], d["dw"], Q.QT2_DTYPE_F32,
                             wsb[name], wsb[name].numel(), cs)

    def e2e_step(i):
        b = i % 2
        B = bufs[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_cmp[b])
            for name, *rest in linears:
                if rest[-1] is None:
                    B[name]["x"].copy_(hosts[name]["x"], non_blocking=True)
                B[name]["dy"].copy_(hosts[name]["dy"], non_blocking=True)
            ev_in[b].record(s_in)
        s_cmp.wait_event(ev_in[b])
        if used[b]:
            s_cmp.wait_event(ev_out[b])
        compute(B, i, s_cmp.cuda_stream)
        ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            for name, *_ in linears:
                for k in ("y", "dx", "dw"):
                    hosts[name][k].copy_(B[name][k], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    flops = step_flops(args.config)
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record(s_in)
    s_cmp.wait_event(e_s)
    s_out.wait_event(e_s)
    n = max(1, min(args.steps, 10))
    for i in range(n):
        e2e_step(100 + i)
    s_in.wait_stream(s_cmp)
    s_in.wait_stream(s_out)
    e_e.record(s_in)
    torch.cuda.synchronize()
    te = max_over_ranks(e_s.elapsed_time(e_e), world, dev)
    e2e = {"value": job_tflops(world, flops, n, te), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": te / n,
           "pipeline": "3 streams (upload, compute, download), 2 device buffer sets; W resident",
           "api": api}

    # the same API calls on resident tensors
    cs = torch.cuda.current_stream(dev)
    for i in range(3):
        compute(bufs[0], i, cs.cuda_stream)
    torch.cuda.synchronize()
    barrier()
    r_s, r_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r_s.record(cs)
    for i in range(n):
        compute(bufs[i % 2], 200 + i, cs.cuda_stream)
    r_e.record(cs)
    torch.cuda.synchronize()
    tr = max_over_ranks(r_s.elapsed_time(r_e), world, dev)
    res = {"value": job_tflops(world, flops, n, tr), "unit": UNIT, "steps": n, "ms_per_step": tr / n,
           "api": api + ", inputs and outputs resident"}
    assert Q.qt2_device_status() == 0
    return e2e, res


# ---------------------------------------------------------------------------------------- oracle
def cpu_baseline(config: str, tokens: int, w_rows: int | None = None, threads: int | None = None):
    """The oracle, as it stands, on a bounded sample of the workload: the full fwd+bwd step of
    the workload's first linear restricted to `tokens` rows of X and dY (a multiple of 128: the
    column views rotate along the tokens) and to the first `w_rows` output features (all when
    None).  Returns (TFLOP/s, seconds, cores, sample)."""
    import oracle as O
    from nvfp4_quantized_b200 import synth

    name, M, K, N, *_ = synth.stack_linears(config)[0]
    x, w, dy = synth.stack_inputs(config, seed=0, only=name)[name]
    Ns = N if w_rows is None else min(N, w_rows)
    xs, dys, w = x[:tokens].contiguous(), dy[:tokens, :Ns].contiguous(), w[:Ns].contiguous()
    O.build()
    old = os.environ.get("QT2_ORACLE_THREADS")
    if threads is not None:
        os.environ["QT2_ORACLE_THREADS"] = str(threads)
    try:
        t0 = time.perf_counter()
        O.linear_fwd(xs, w)
        O.linear_bwd(dys, xs, w, seed=1)
        dt = time.perf_counter() - t0
        cores = O.threads()
    finally:
        if threads is not None:
            if old is None:
                os.environ.pop("QT2_ORACLE_THREADS", None)
            else:
                os.environ["QT2_ORACLE_THREADS"] = old
    flops = 3 * 2.0 * tokens * Ns * K
    sample = (f"full fwd+bwd of the '{name}' linear ({K} -> {N}) on {tokens} of {M} tokens and {Ns} of {N} output "
              f"features (X, dY rows; W {Ns}x{K}); oracle fp64 GEMMs and bit-exact quantizers")
    return flops / dt / 1e12, dt, cores, sample


# ---------------------------------------------------------------------------------------- sweep
def run_sweep(args):
    """Both quantizers alone: 2^20..2^30 elements as rows of 2048 / 4096 / 14336, the forward
    quantizer (row view) and MS-EDEN (ROW, COL, BOTH); CUDA events per call, L2 flushed by a
    256 MiB write between calls; median of --steps calls after --warmup."""
    import torch
    from nvfp4_quantized_b200 import build as qbuild
    from nvfp4_quantized_b200 import qt2 as Q, synth
    qbuild.build()
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    pk = peaks()
    points = []
    for L in (2048, 4096, 14336):
        for p in range(20, 31):
            R = synth.sweep_rows(p, L)
            x = synth.sweep_tensor(p, L, seed=p, device=dev)
            n = R * L
            vr, vc = Q.alloc_view(R, L, dev), Q.alloc_view(L, R, dev)
            ws = Q.alloc_workspace(max(Q.qt2_quant_msedEN_workspace_size(R, L, Q.QT2_LAYOUT_BOTH),
                                       Q.qt2_quant_fwd46_workspace_size(R, L)), dev)
            calls = {("fwd46", "ROW"): (lambda: Q.qt2_quant_fwd46(x, R, L, L, Q.QT2_LAYOUT_ROW, vr, None, ws,
                                                                   ws.numel(), st), n * BYTES_FWD46)}
            for mask, tag, b in ((Q.QT2_LAYOUT_ROW, "ROW", BYTES_MSED_ONE), (Q.QT2_LAYOUT_COL, "COL", BYTES_MSED_ONE),
                                 (Q.QT2_LAYOUT_BOTH, "BOTH", BYTES_MSED_BOTH)):
                calls[("msedEN", tag)] = (
                    lambda mask=mask: Q.qt2_quant_msedEN(x, R, L, L, mask, 7, 1, 2, vr if mask & 1 else None,
                                                         vc if mask & 2 else None, ws, ws.numel(), st), n * b)
            for (q, view), (fn, nbytes) in calls.items():
                for _ in range(args.warmup):
                    fn()
                ts = []
                for _ in range(args.steps):
                    flush.fill_(1)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(st)
                    fn()
                    b.record(st)
                    torch.cuda.synchronize()
                    ts.append(a.elapsed_time(b))
                ms = sorted(ts)[len(ts) // 2]
                gbs = nbytes / (ms * 1e-3) / 1e9
                points.append({"quantizer": q, "view": view, "row_length": L, "rows": R, "elements": n,
                               "log2_elements": p, "ms": ms, "gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"]})
            assert Q.qt2_device_status(st) == 0
            del x, vr, vc, ws
            torch.cuda.empty_cache()
    print(json.dumps({"mode": "sweep", "metric": "quantizer GB/s (algorithmic bytes) and fraction of HBM",
                      "unit": "GB/s", "peak_gbs": pk["hbm_gbs"], "peak_source": pk["source"],
                      "timing": f"median of {args.steps} calls after {args.warmup}, L2 flushed between calls",
                      "data": "synthetic: N(0,1) with 0.1% of elements x50", "points": points}), flush=True)


def run_op(args):
    """--op fwd46_sq: the square-block weight quantizer on the config's first W [N][K] (both
    views), timed alone with CUDA events (two W inputs alternate)."""
    import torch
    from nvfp4_quantized_b200 import build as qbuild
    from nvfp4_quantized_b200 import qt2 as Q, synth
    qbuild.build()
    dev = torch.device("cuda", 0)
    name, M, K, N, *_ = synth.stack_linears(args.config)[0]
    ws_ = [synth.stack_inputs(args.config, seed=10 * i, device=dev)[name][1] for i in range(2)]
    vr, vc = Q.alloc_view(N, K, dev), Q.alloc_view(K, N, dev)
    ws = Q.alloc_workspace(Q.qt2_quant_fwd46_sq_workspace_size(N, K), dev)
    st = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        Q.qt2_quant_fwd46_sq(ws_[i % 2], N, K, K, vr, vc, ws, ws.numel(), st)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(args.steps):
        Q.qt2_quant_fwd46_sq(ws_[i % 2], N, K, K, vr, vc, ws, ws.numel(), st)
    e1.record(st)
    torch.cuda.synchronize()
    assert Q.qt2_device_status(st) == 0
    ms = e0.elapsed_time(e1) / args.steps
    gbs = N * K * BYTES_FWD46_SQ / (ms * 1e-3) / 1e9
    pk = peaks()
    print(json.dumps({"op": "qt2_quant_fwd46_sq", "metric": "square-block quantizer GB/s (algorithmic bytes)",
                      "value": gbs, "unit": "GB/s", "ms_per_call": ms, "hbm_frac": gbs / pk["hbm_gbs"],
                      "steps": args.steps, "warmup": args.warmup,
                      "config": {"tensor": f"W {N}x{K} bf16", "views": "row [N][K] and column [K][N]"}}),
          flush=True)


# ---------------------------------------------------------------------------------------- main
def workload_name(config: str) -> str:
    from nvfp4_quantized_b200 import synth
    parts = ", ".join(f"{n} {K}->{N}" for n, M, K, N, *_ in synth.stack_linears(config))
    M = synth.stack_linears(config)[0][1]
    desc = {"mlp8b": "Llama-3-8B MLP (gate, up, down)", "stack1p1b": "1.1B-class block linears (QKV, O, gate, "
            "up, down)", "llm1p9b": "1.9B-class linear", "mlp8b_up": "Llama-3-8B MLP up projection",
            "mlp8b_down": "Llama-3-8B MLP down projection"}.get(config, config)
    return (f"Quartet II NVFP4 linear layers fwd+bwd (forward RTN+4/6, backward MS-EDEN, 3 block-scaled GEMMs "
            f"each): {desc} at {M} tokens: {parts}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="mlp8b",
                    choices=["mlp8b", "stack1p1b", "llm1p9b", "mlp8b_up", "mlp8b_down"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-torch", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=128)
    ap.add_argument("--ref-w-rows", type=int, default=2048)
    # the oracle's samples: about 10 s of host work each (all cores; one thread)
    ap.add_argument("--cpu-tokens", type=int, default=1024)
    ap.add_argument("--cpu-w-rows", type=int, default=8192)
    ap.add_argument("--cpu-tokens-1t", type=int, default=256)
    ap.add_argument("--cpu-w-rows-1t", type=int, default=3072)
    ap.add_argument("--schedule", choices=["onepass", "separate", "fused", "local"], default="onepass",
                    help="onepass (default): every tensor quantized once a step, both of its views from one read "
                         "(qt2_quant_fwd46_msedEN_col on X and on W; MS-EDEN of dY, both views); separate: each "
                         "linear as qt2_linear_fwd/bwd runs it (one quantizer call per view, X per linear); "
                         "fused: X's forward and column views from one read (qt2_quant_fwd46_msedEN_col) and "
                         "W's forward and column views made once and reused by every step, as micro-batches of "
                         "one optimizer step; local: the forward with CTA-local scales (qt2_quant_fwd46_local, "
                         "qt2_gemm_nvfp4_local), a different numeric contract")
    ap.add_argument("--op", choices=["fwd46_sq"], default=None,
                    help="time one library call alone instead of the layer step")
    ap.add_argument("--sweep", action="store_true", help="the quantizer sweep over sizes, row lengths and views")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.op:
        return run_op(args)
    if args.sweep:
        return run_sweep(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    workload = workload_name(args.config)
    flops = step_flops(args.config)

    if args.impl == "reference":
        if rank != 0:
            return
        steps = []
        for i in range(args.warmup + args.steps):
            v, dt, cores, sample = cpu_baseline(args.config, args.ref_tokens, args.ref_w_rows)
            if i >= args.warmup:
                steps.append((v, dt))
        value = sum(v for v, _ in steps) / len(steps)
        ms = 1e3 * sum(dt for _, dt in steps) / len(steps)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64 (GEMM), f32 (quantizers)",
                "data": "synthetic", "config": {"workload": workload, "sample_tokens": args.ref_tokens},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    from nvfp4_quantized_b200 import build as qbuild
    if rank == 0:
        qbuild.build()
    if world > 1:
        dist.barrier()

    r = run_ours(args, rank, world, local_rank)
    pk = peaks()
    value = job_tflops(world, flops, args.steps, r["max_ms"])
    lin = {n: (M, K, N) for n, M, K, N, *_ in r["linears"]}

    kernels, gemm_ms, gemm_flops, q_ms, q_bytes = {}, 0.0, 0.0, 0.0, 0.0
    for (ln, call), ms in zip(r["names"], r["per"]):
        kind, work = call_work(call, *lin[ln])
        key = f"{ln}.{call}" if len(lin) > 1 else call
        if kind == "gemm":
            t = work / (ms * 1e-3) / 1e12
            kernels[key] = {"ms": ms, "tflops": t, "fp4_frac": t / (pk["bf16"] * FP4_PER_BF16)}
            gemm_ms, gemm_flops = gemm_ms + ms, gemm_flops + work
        else:
            g = work / (ms * 1e-3) / 1e9
            kernels[key] = {"ms": ms, "gbs": g, "hbm_frac": g / pk["hbm_gbs"]}
            q_ms, q_bytes = q_ms + ms, q_bytes + work
    fp4_peak = pk["bf16"] * FP4_PER_BF16
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    traffic = gemm_traffic(args.config)
    n_gemm = sum(1 for _, c in r["names"] if c.startswith("gemm_"))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["max_ms"] / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x ue4m3 block-scaled GEMM, fp32 accumulate; fp32 quantizers)",
        "data": "synthetic (seeded bf16 tensors with the layers' distributions)",
        "config": {"workload": workload, "name": args.config,
                   "linears": [{"name": n, "M": M, "K": K, "N": N, "shares_x_with": s}
                               for n, M, K, N, _, _, s in r["linears"]],
                   "flop_per_step": flops,
                   "parallelism": f"dp{world}: every rank its own token batch, no collective on the path",
                   "l2": "inputs larger than L2: every step reads several GB, two input sets alternate",
                   "output": "Y bf16, dX bf16, dW fp32", "schedule": args.schedule,
                   "schedule_calls": SCHEDULE_NOTE[args.schedule]},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp4_peak, "traffic": traffic,
                     "kernel": f"gemm_nvfp4_pair_kernel (all {n_gemm} GEMM launches of the step: their FLOPs over "
                               "their summed event time)",
                     "peak_source": f"{pk['source']}: burst bf16 {pk['bf16']} TFLOP/s x {FP4_PER_BF16:g} (nominal "
                                    "dense fp4/bf16 ratio); each GEMM is event-timed as one launch",
                     "frac_of_sustained": achieved / (pk["bf16_sustained"] * FP4_PER_BF16)},
        "quantizers": {"gbs": q_bytes / (q_ms * 1e-3) / 1e9, "hbm_frac": q_bytes / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                       "peak_gbs": pk["hbm_gbs"], "ms_per_step": q_ms, "bytes_per_step": q_bytes},
        "gemm_ms_per_step": gemm_ms,
        "kernels": kernels,
        "gpu_launches": r["launches"],
        "gpu_launches_source": "kernel launches of libqt2.so in the timed region, counted through qt2_set_fault_hook",
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if r["torch"] is not None:
        t = r["torch"]
        t["gemm_speedup"] = t["ms_per_step"] / gemm_ms
        t["step_speedup"] = t["ms_per_step"] / (r["max_ms"] / args.steps)
        line["torch_bf16"] = t
    if r["e2e"] is not None:
        line["e2e"] = r["e2e"]
        line["e2e_resident"] = r["e2e_resident"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, cores, sample = cpu_baseline(args.config, args.cpu_tokens, args.cpu_w_rows)
        v1, dt1, _, sample1 = cpu_baseline(args.config, args.cpu_tokens_1t, args.cpu_w_rows_1t, threads=1)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                                "seconds": dt,
                                "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "sample": sample1,
                                                  "seconds": dt1}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def gemm_traffic(config: str):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken on this config
    and on the current kernel source (else None)."""
    prof = os.path.join(ROOT, "profiles", "gemm_nvfp4_traffic.json")
    if not os.path.exists(prof):
        return None
    try:
        import hashlib
        with open(prof) as f:
            tj = json.load(f)
        src = os.path.join(ROOT, "nvfp4_quantized_b200", "csrc", "gemm2_kernel.cuh")
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        if tj.get("config") == config and tj.get("kernel_sha1") == sha:
            return tj.get("bytes_per_launch")
    except Exception:
        return None
    return None


if __name__ == "__main__":
    main()
