"""Benchmark of HSTU causal pointwise aggregated attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path over one batch of synthetic input:
for the forward workloads the fused attention + LayerNorm + gate forward, for
the training workloads the forward with saved statistics followed by the
backward.  The default workload is the jagged one: 64 sequences of 256..4096
tokens (seed 0), 8 heads, d_qk = d_v = 128, position and time bias,
normalisation by each sequence's own length, bf16 -- the largest
configuration that fits one GPU.  After the main line's measurement the
long-sequence forward and the training step are timed as well (``also``).

Timing: inputs are resident in HBM; R input sets whose total size exceeds
twice the 126 MB L2 are used in rotation, so no step reads its inputs from L2
left by the previous one.  The steps are replayed from a CUDA graph (no host
work inside the timed region), bracketed by a barrier and a device
synchronisation on both sides and timed with CUDA events on the launching
stream; the maximum over ranks is reported.  Under torchrun every rank runs
its own batch (independent sequences, no collective on the data path: weak
scaling), and `value` counts the FLOPs of all ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hstu_inputs as hi  # noqa: E402

METRIC = "causal HSTU-attention TFLOP/s (bf16) and % of B200 dense tensor peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FWD_KERNEL = "hstu_fwd_bf16_sm100"
BWD_KERNELS = "bwd_pre_rows_bf16, hstu_bwd_dq_sm100, hstu_bwd_dkdv_sm100"
KERNEL_SOURCES = {
    "hstu_fwd_bf16_sm100": ["pointwise_attention_b200/csrc/fwd_sm100.cu",
                            "pointwise_attention_b200/csrc/ptx.cuh",
                            "pointwise_attention_b200/csrc/tile_math.cuh",
                            "pointwise_attention_b200/csrc/bounds.cuh",
                            "pointwise_attention_b200/csrc/internal.h"],
}
BWD_FLOP_FACTOR = 2.5      # S recomputed, dA, dV, dQ, dK: five GEMM-equivalents


# ----------------------------------------------------------------- host logic
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch of independent sequences."""
    return base_seed + 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_bytes(inp) -> int:
    """Bytes a launch must move at least: read Q, K, V, U, the bias tables,
    timestamps and offsets once; write Y once."""
    es = 2 if inp.spec.dtype == "bf16" else 4
    T, H = inp.q.shape[0], inp.q.shape[1]
    # q, k [T,H,dqk]; v [T,H,dv]; u and y [T,H*dv]
    n = T * H * (2 * inp.q.shape[2] + inp.v.shape[2]) * es + 2 * T * H * inp.v.shape[2] * es
    if inp.rab_pos is not None:
        n += inp.rab_pos.numel() * 4
    if inp.rab_time is not None:
        n += inp.rab_time.numel() * 4 + T * 8
    n += inp.offsets.numel() * 4
    return int(n)


def set_bytes(inp, train: bool) -> int:
    """Device bytes of one input set (plus the training step's saved outputs
    and gradients)."""
    n = algorithmic_bytes(inp)
    if train:
        n += inp.total_tokens * inp.q.shape[1] * inp.v.shape[2] * (4 + 2 * 5)
    return n


def n_sets(inp, train: bool) -> int:
    """Input sets in rotation: together more than twice the L2."""
    return max(2, int(math.ceil(2 * L2_BYTES / set_bytes(inp, train))))


def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "%s.%s.txt" % (kernel, workload))
    srcs = KERNEL_SOURCES.get(kernel)
    if not os.path.exists(path) or not srcs:
        return None
    fields = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("kernel_source_sha256") != source_digest(srcs):
        return None
    try:
        return int(float(fields["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_threads() -> int:
    """Threads the oracle's OpenMP runtime uses by default: the CPUs this
    process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed region."""

    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.period = [], set(), period_s
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:   # NVML unavailable: report no clocks rather than guess
            self.nv = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nv is not None:
            self.t.join()
            if not self.samples:
                self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def bench_config(spec, inp, world: int) -> dict:
    """The `config` object of both arms: the workload and how its inputs
    relate to the L2 between steps (`inp` is rank 0's drawn problem)."""
    c = {"workload": spec.name, "batch": spec.batch, "heads": spec.heads, "d_qk": spec.d_qk,
         "d_v": spec.d_v,
         "rab": "+".join(x for x, on in (("pos", spec.rab_pos_len > 0), ("time", spec.rab_time))
                         if on) or "none",
         "norm": "own_length" if spec.norm == "own" else "fixed"}
    if spec.len_range:
        c["seq_len"] = "U[%d,%d]" % spec.len_range
    else:
        c["seq_len"] = spec.seq_len
    if spec.stochastic_length:
        c["stochastic_length"] = "keep %d, p %.2f" % spec.stochastic_length
    c["parallelism"] = "replicas" if world > 1 else "single"
    R = n_sets(inp, spec.grad)
    c["l2"] = "%d rotating input sets (%.0f MB each) > 2x 126 MB L2" % (
        R, set_bytes(inp, spec.grad) / 1e6)
    return c


# ----------------------------------------------------------------- oracle arm
def _row_sample(inp, nrows: int, seed: int = 0):
    """nrows token rows drawn uniformly (seeded, without replacement) over the
    whole packed token axis, and their forward FLOPs.  Row i of a sequence
    costs i + 1 columns, so a uniform sample keeps the workload's mix of short
    and long rows and its FLOP rate stands for the whole."""
    import numpy as np
    T = inp.total_tokens
    nrows = max(1, min(int(nrows), T))
    g = torch.Generator().manual_seed(seed)
    rows = torch.randperm(T, generator=g)[:nrows].sort().values.numpy().astype(np.int64)
    offs = inp.offsets.numpy()
    seq = np.searchsorted(offs, rows, side="right") - 1
    local = rows - offs[seq]
    H, dqk, dv = inp.q.shape[1], inp.q.shape[2], inp.v.shape[2]
    fl = int(2 * (local + 1).sum() * H * (dqk + dv))
    return rows, fl


def oracle_step_sample(inp, budget_s: float, threads: int):
    """Times the oracle forward on `threads` host threads: the whole workload
    if it fits in the budget, else a uniform random sample of its rows sized
    from a small probe; returns (flops, seconds, description, extrapolated)."""
    import oracle
    oracle.build()
    flops_full = hi.causal_flops(inp.lengths, inp.q.shape[1], inp.q.shape[2], inp.v.shape[2])
    per_row = flops_full / max(inp.total_tokens, 1)
    rows, fl = _row_sample(inp, math.ceil((2e9 if threads > 1 else 2e8) / per_row), seed=1)
    t0 = time.perf_counter()
    oracle.fwd_rows(inp, rows, threads=threads)
    rate = fl / max(time.perf_counter() - t0, 1e-9)
    if flops_full / rate <= budget_s:
        reps, total = 0, 0.0
        while reps == 0 or total < budget_s * 0.5:
            t0 = time.perf_counter()
            oracle.fwd(inp, threads=threads)
            total += time.perf_counter() - t0
            reps += 1
        return flops_full * reps, total, "full workload forward x%d" % reps, False
    rows, fl = _row_sample(inp, math.ceil(rate * budget_s / per_row), seed=2)
    t0 = time.perf_counter()
    oracle.fwd_rows(inp, rows, threads=threads)
    return fl, time.perf_counter() - t0, (
        "%d token rows drawn uniformly from the workload's %d (forward, every head)"
        % (len(rows), inp.total_tokens)), True


def cpu_baseline(inp, budget_all: float, budget_single: float) -> dict:
    """The oracle on all host threads and on one, each on a bounded sample of
    the workload; the full workload's time is extrapolated from the sample's
    FLOP rate where only a sample was run."""
    threads = host_threads()
    flops_full = hi.causal_flops(inp.lengths, inp.q.shape[1], inp.q.shape[2], inp.v.shape[2])
    f, s, desc, ext = oracle_step_sample(inp, budget_all, threads)
    out = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
           "sample": desc, "cpu_model": cpu_model(),
           ("full_forward_s_extrapolated" if ext else "full_forward_s"): flops_full / (f / s)}
    f1, s1, desc1, ext1 = oracle_step_sample(inp, budget_single, 1)
    out["single_thread"] = {
        "value": f1 / s1 / 1e12, "unit": "TFLOP/s", "sample": desc1,
        ("full_forward_s_extrapolated" if ext1 else "full_forward_s"): flops_full / (f1 / s1)}
    return out


def run_reference(args, spec):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = hi.make_inputs(spec, seed=args.seed)
    threads = host_threads()
    for _ in range(args.warmup):
        oracle_step_sample(inp, 0.5, threads)
    flops, secs = 0, 0.0
    desc = ""
    for _ in range(args.steps):
        f, s, desc, _ = oracle_step_sample(inp, args.ref_step_budget, threads)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(spec, inp, world),
        "timing": "host wall clock around each sampled oracle forward",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm
class Workload:
    """R device copies of one rank's inputs plus outputs and workspaces."""

    def __init__(self, inp, train: bool, device):
        import pointwise_attention_b200 as pa
        self.pa, self.inp, self.train = pa, inp, train
        self.R = n_sets(inp, train)
        self.sets = []
        for _ in range(self.R):
            d = {k: (None if v is None else v.to(device).contiguous()) for k, v in dict(
                q=inp.q, k=inp.k, v=inp.v, u=inp.u, offsets=inp.offsets, ts=inp.timestamps,
                rab_pos=inp.rab_pos, rab_time=inp.rab_time, dy=inp.dy).items()}
            T, H, dv = inp.q.shape[0], inp.q.shape[1], inp.v.shape[2]
            d["y"] = torch.empty((T, H * dv), dtype=inp.q.dtype, device=device)
            p = pa.make_problem(d["q"], d["v"], d["offsets"], inp.max_seq_len, d["ts"],
                                d["rab_pos"], d["rab_time"], inp.norm_len)
            d["ws"] = pa.new_workspace(p, train, device)
            if train:
                d["saved"] = (torch.empty((T, H * dv), dtype=torch.float32, device=device),
                              torch.empty((T,), dtype=torch.float32, device=device),
                              torch.empty((T,), dtype=torch.float32, device=device))
                d["grads"] = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]),
                                  dv=torch.empty_like(d["v"]), du=torch.empty_like(d["u"]),
                                  d_rab_pos=(torch.empty_like(d["rab_pos"])
                                             if d["rab_pos"] is not None else None),
                                  d_rab_time=(torch.empty_like(d["rab_time"])
                                              if d["rab_time"] is not None else None))
            self.sets.append(d)
        # forward (after the time-plan pass with a bf16 time table); the
        # backward's LN/gate kernel, its time-plan pass, dQ and dK/dV kernels
        plans = 1 if (inp.q.dtype == torch.bfloat16 and inp.rab_time is not None) else 0
        self.launches_per_step = (1 + plans) if not train else (1 + plans) + (3 + plans)

    def forward(self, i: int, stream=None):
        d, inp, pa = self.sets[i % self.R], self.inp, self.pa
        pa.hstu_attn_fwd(d["q"], d["k"], d["v"], d["u"], d["offsets"], inp.max_seq_len,
                         timestamps=d["ts"], rab_pos=d["rab_pos"], rab_time=d["rab_time"],
                         norm_len=inp.norm_len, save_for_backward=self.train, y=d["y"],
                         saved=d.get("saved"), workspace=d["ws"], stream=stream)

    def backward(self, i: int, stream=None):
        d, inp, pa = self.sets[i % self.R], self.inp, self.pa
        pa.hstu_attn_bwd(d["dy"], d["q"], d["k"], d["v"], d["u"], d["offsets"],
                         inp.max_seq_len, d["saved"], timestamps=d["ts"],
                         rab_pos=d["rab_pos"], rab_time=d["rab_time"],
                         norm_len=inp.norm_len, grads=d["grads"], workspace=d["ws"],
                         stream=stream)

    def step(self, i: int, stream=None):
        self.forward(i, stream)
        if self.train:
            self.backward(i, stream)

    def check(self):
        for d in self.sets:
            rc = self.pa.hstu_attn_check(d["ws"])
            if rc != 0:
                raise RuntimeError("device status after the timed region: %s"
                                   % self.pa.status_string(rc))


def graph_of(fn, count: int, stream):
    """CUDA graph of fn(0) .. fn(count-1) on `stream`."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(count):
                fn(i, stream=stream)
    torch.cuda.synchronize()
    return g


def time_graphs(steps: int, R: int, fn, stream, world: int, clock_index=None):
    """Replays graphs of R steps (plus a tail graph) until exactly `steps` steps
    ran; returns (seconds on the device, max over ranks, clock summary)."""
    reps, rest = divmod(steps, R)
    graph = graph_of(fn, R, stream)
    tail = graph_of(fn, rest, stream) if rest else None
    for _ in range(2):                      # graph warm-up
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(clock_index) if clock_index is not None else None
    if clk is not None:
        clk.__enter__()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        if tail is not None:
            tail.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if clk is not None:
        clk.__exit__(None, None, None)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    elapsed = e0.elapsed_time(e1) / 1e3
    return elapsed, clk.summary() if clk is not None else None


def measure(spec, seed: int, steps: int, warmup: int, device, world: int, local: int,
            clocks: bool):
    """Times `steps` steps of one workload; returns the measurement and the
    Workload (for the end-to-end leg)."""
    inp = hi.make_inputs(spec, seed=seed)
    train = spec.grad
    wl = Workload(inp, train, device)
    flops_fwd = hi.causal_flops(inp.lengths, spec.heads, spec.d_qk, spec.d_v)
    flops_step = flops_fwd * (1 + (BWD_FLOP_FACTOR if train else 0.0))
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    wl.check()

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        wl.step(0, stream=stream)           # warm the capture stream
    torch.cuda.synchronize()
    elapsed, clk = time_graphs(steps, wl.R, wl.step, stream, world,
                               local if clocks else None)
    elapsed_max = reduce_max(elapsed, world, device)
    wl.check()
    peaks, peak_kind = load_peaks()
    res = {"inp": inp, "flops_fwd": flops_fwd, "flops_step": flops_step,
           "elapsed": elapsed, "elapsed_max": elapsed_max, "clocks": clk,
           "value": flops_step * steps * world / elapsed_max / 1e12,
           "ms_per_step": elapsed_max / steps * 1e3, "launches_per_step": wl.launches_per_step}

    if not train:
        # One forward launch per step, replayed back to back from the graph:
        # the average launch duration is the timed region over the steps.
        t_launch = elapsed / steps
        bytes_launch = algorithmic_bytes(inp)
        t_hbm = bytes_launch / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops_fwd / (peaks["bf16_tflops"] * 1e12)
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": bytes_launch / t_launch / 1e9,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        else:
            roof = {"bound": "tensor", "achieved": flops_fwd / t_launch / 1e12,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = profiled_traffic(FWD_KERNEL, spec.name)
        roof["peak_source"] = peak_kind + (" burst" if roof["bound"] == "tensor" else "")
        roof["kernel"] = FWD_KERNEL if spec.dtype == "bf16" else "fwd_simt<float>"
        roof["algorithmic_bytes"] = bytes_launch
        roof["algorithmic_flops"] = flops_fwd
        roof["us_per_launch"] = t_launch * 1e6
    else:
        # Training: the backward call (LN/gate, dQ and dK/dV kernels) is the
        # dominant unit.  It is timed on its own: graphs of R backward calls,
        # replayed, on the saved outputs the timed steps left behind.
        bsteps = max(wl.R, steps)
        t_b, _ = time_graphs(bsteps, wl.R, wl.backward, stream, world)
        t_bwd = t_b / bsteps
        flops_bwd = BWD_FLOP_FACTOR * flops_fwd
        roof = {"bound": "tensor", "achieved": flops_bwd / t_bwd / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = None
        roof["peak_source"] = peak_kind + " burst"
        roof["kernel"] = "hstu_attn_bwd (%s)" % (
            BWD_KERNELS if inp.rab_time is None else BWD_KERNELS + ", time_plans")
        roof["algorithmic_flops"] = flops_bwd
        roof["ms_per_call"] = t_bwd * 1e3
        roof["flops_2x_fwd_tflops"] = 2.0 * flops_fwd / t_bwd / 1e12
        wl.check()
    res["roofline"] = roof
    return res, wl


def timed_e2e(wl, steps: int, device):
    """Same step through the public API with host buffers: H2D copy of the
    step's inputs from pinned memory, the call, D2H copy of the result."""
    inp, d = wl.inp, wl.sets[0]
    names = ["q", "k", "v", "u", "offsets"] + [n for n in ("ts", "rab_pos", "rab_time") if
                                               d[n] is not None]
    if wl.train:
        names.append("dy")
    src = dict(q=inp.q, k=inp.k, v=inp.v, u=inp.u, offsets=inp.offsets, ts=inp.timestamps,
               rab_pos=inp.rab_pos, rab_time=inp.rab_time, dy=inp.dy)
    host = {n: src[n].contiguous().pin_memory() for n in names}
    # The step's result: Y for a forward step, the input gradients for a training step.
    outs = ([d["grads"][n] for n in ("dq", "dk", "dv", "du")] if wl.train else [d["y"]])
    out_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host)
    stream = torch.cuda.current_stream()

    def one():
        for n in names:
            d[n].copy_(host[n], non_blocking=True)
        wl.step(0)
        for dst, src_t in zip(out_host, outs):
            dst.copy_(src_t, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3, h2d, d2h


def measure_proj(T: int, steps: int, device, world: int):
    """The projections around the attention at the model card's block shape
    (embed 512, 4 heads, d = 128): UVQK (+ bias, SiLU) and the output
    projection + residual + LayerNorm, each timed alone (CUDA graph of R
    calls, events on the launching stream)."""
    import pointwise_attention_b200 as pa
    peaks, peak_kind = load_peaks()
    E, H, d = 512, 4, 128
    N, D = 4 * H * d, H * d
    # enough copies that one graph's operands exceed the 126 MB L2
    per_set = T * (E + N + D + E) * 2
    R = max(2, -(-256 * 2 ** 20 // per_set))
    sets = []
    for r in range(R):
        p = hi.make_proj_inputs(T, E, H, d, d, seed=100 + r)
        dd = {k: getattr(p, k).to(device) for k in ("x", "w_uvqk", "b_uvqk", "y", "w_out",
                                                    "b_out", "ln_weight", "ln_bias")}
        dd["out"] = pa.hstu_uvqk_fwd(dd["x"], dd["w_uvqk"], H, d, d, bias=dd["b_uvqk"], act=1)
        dd["z"], _ = pa.hstu_out_fwd(dd["y"], dd["w_out"], dd["x"], bias=dd["b_out"],
                                     ln_weight=dd["ln_weight"], ln_bias=dd["ln_bias"])
        dd["ws"] = torch.zeros(256, dtype=torch.uint8, device=device)
        sets.append(dd)

    def uvqk(i, stream=None):
        dd = sets[i % R]
        pa.hstu_uvqk_fwd(dd["x"], dd["w_uvqk"], H, d, d, bias=dd["b_uvqk"], act=1,
                         out=dd["out"], workspace=dd["ws"], stream=stream)

    def out(i, stream=None):
        dd = sets[i % R]
        pa.hstu_out_fwd(dd["y"], dd["w_out"], dd["x"], bias=dd["b_out"],
                        ln_weight=dd["ln_weight"], ln_bias=dd["ln_bias"], z=dd["z"],
                        workspace=dd["ws"], stream=stream)

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    result = {"workload": "proj_E512_H4_d128_T%d" % T, "steps_timed": steps}
    for name, fn, flops, nbytes, kern in (
            ("uvqk", uvqk, 2.0 * T * E * N, T * (E + N) * 2 + N * E * 2, "proj_gemm_sm100<0,256>"),
            ("out", out, 2.0 * T * D * E, T * (D + 2 * E) * 2 + E * D * 2,
             "proj_gemm_sm100<1,512>")):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        t, _ = time_graphs(steps, R, fn, stream, world)
        t = reduce_max(t, world, device) / steps
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
        if t_tc >= t_hbm:
            roof = {"bound": "tensor", "achieved": flops / t / 1e12, "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s"}
        else:
            roof = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s"}
        roof.update(frac=roof["achieved"] / roof["peak"], kernel=kern, peak_source=peak_kind,
                    algorithmic_flops=flops, algorithmic_bytes=nbytes, us_per_launch=t * 1e6,
                    tflops=flops / t / 1e12, traffic=None)
        for s_ in sets:
            if pa.hstu_attn_check(s_["ws"]) != 0:
                raise RuntimeError("device status after the projection timing")
        result[name] = roof
    return result


def measure_cand(name: str, steps: int, device, world: int, seed: int):
    """Candidate scoring against cached histories (M-FALCON reading) on the
    named candidate workload, one call per step from a CUDA graph (the
    histories' keys and values, over 300 MB, exceed the L2)."""
    import ctypes
    import pointwise_attention_b200 as pa
    peaks, peak_kind = load_peaks()
    sp, ncand = hi.CAND_WORKLOADS[name]
    ci = hi.make_cand_inputs(sp, ncand, seed=seed)
    h = ci.hist
    d = lambda t: None if t is None else t.to(device)
    args = [d(h.k), d(h.v), d(h.offsets), max(h.lengths), d(ci.qc), d(ci.kc), d(ci.vc),
            d(ci.uc), d(ci.cand_offsets), max(ci.counts)]
    kw = dict(timestamps=d(h.timestamps), cand_timestamps=d(ci.cand_ts), rab_pos=d(h.rab_pos),
              rab_time=d(h.rab_time), norm_len=h.norm_len)
    p = pa.make_problem(args[0], args[1], args[2], args[3], kw["timestamps"], kw["rab_pos"],
                        kw["rab_time"], h.norm_len)
    n = pa.load_library().hstu_cand_workspace_size(ctypes.byref(p), ci.total_cands,
                                                    max(ci.counts))
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    y = pa.hstu_cand_fwd(*args, workspace=ws, **kw)

    def fn(i, stream=None):
        pa.hstu_cand_fwd(*args, y=y, workspace=ws, stream=stream, **kw)

    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    t, _ = time_graphs(steps, 1, fn, stream, world)
    t = reduce_max(t, world, device) / steps
    if pa.hstu_attn_check(ws) != 0:
        raise RuntimeError("device status after the candidate-scoring timing")
    # each candidate: n_b history keys and itself, H heads, d_qk + d_v
    flops = 2.0 * sum(c * (nb + 1) for c, nb in zip(ci.counts, h.lengths)) * sp.heads * (
        sp.d_qk + sp.d_v)
    roof = {"bound": "tensor", "achieved": flops / t / 1e12, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "kernel": "hstu_cand_sm100", "peak_source": peak_kind + " burst",
            "algorithmic_flops": flops, "us_per_launch": t * 1e6, "traffic": None}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return {"workload": name, "users": sp.batch, "candidates_per_user": ncand,
            "history_tokens": h.total_tokens, "value": roof["achieved"], "unit": "TFLOP/s",
            "ms_per_step": t * 1e3, "steps_timed": steps, "roofline": roof}


def summary_of(spec, res, world):
    roof = dict(res["roofline"])
    return {"workload": spec.name, "value": res["value"], "unit": "TFLOP/s",
            "ms_per_step": res["ms_per_step"], "steps_timed": res["steps"],
            "pct_of_dense_bf16_peak": 100.0 * res["value"] / world / roof["peak"],
            "roofline": roof}


def run_gpu(args, spec):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=device)
    import pointwise_attention_b200 as pa
    pa.load_library()

    res, wl = measure(spec, rank_seed(args.seed, rank), args.steps, args.warmup, device, world,
                      local, clocks=True)
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    e2e_t, h2d, d2h = timed_e2e(wl, e2e_steps, device)
    e2e_t = reduce_max(e2e_t, world, device)
    inp = res["inp"]
    del wl

    also = {}
    for name in [x for x in args.also.split(",") if x and x != spec.name]:
        if name == "proj":
            also[name] = measure_proj(131072, args.also_steps, device, world)
            torch.cuda.empty_cache()
            continue
        if name in hi.CAND_WORKLOADS:
            also[name] = measure_cand(name, args.also_steps, device, world,
                                      rank_seed(args.seed, rank))
            torch.cuda.empty_cache()
            continue
        sp = hi.WORKLOADS[name]
        steps = args.also_steps
        r2, wl2 = measure(sp, rank_seed(args.seed, rank), steps, 3, device, world, local,
                          clocks=False)
        r2["steps"] = steps
        del wl2
        torch.cuda.empty_cache()
        also[name] = summary_of(sp, r2, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_budget, args.cpu_budget_single)

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    roof = res["roofline"]
    line = {
        "metric": METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if spec.dtype == "bf16" else "f32", "data": "synthetic",
        "pct_of_dense_bf16_peak": 100.0 * res["value"] / world / roof["peak"],
        "config": bench_config(spec, inp, world),
        "timing": "CUDA graph of %d steps replayed, CUDA events on the launching stream" % (
            n_sets(inp, spec.grad)),
        "gpu_launches": args.steps * res["launches_per_step"],
        "roofline": roof,
        "cpu_baseline": cpu,
        "clocks": res["clocks"],
    }
    line["e2e"] = {"value": res["flops_step"] * world * e2e_steps / e2e_t / 1e12,
                   "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "steps": e2e_steps}
    if also:
        line["also"] = also
    print(json.dumps(line), flush=True)
    return 0


def run_once(args, spec):
    """One call of the forward, the backward or candidate scoring (the mfalcon
    workload), run twice on one input set: the launch a profiler captures
    (ncu -s 1 -c 1), with nothing around it."""
    import pointwise_attention_b200 as pa
    torch.cuda.set_device(0)
    if args.once == "cand":
        sp, ncand = hi.CAND_WORKLOADS["mfalcon"]
        ci = hi.make_cand_inputs(sp, ncand, seed=args.seed)
        h = ci.hist
        d = lambda t: None if t is None else t.to("cuda").contiguous()
        cargs = [d(h.k), d(h.v), d(h.offsets), max(h.lengths), d(ci.qc), d(ci.kc), d(ci.vc),
                 d(ci.uc), d(ci.cand_offsets), max(ci.counts)]
        ckw = dict(timestamps=d(h.timestamps), cand_timestamps=d(ci.cand_ts),
                   rab_pos=d(h.rab_pos), rab_time=d(h.rab_time), norm_len=h.norm_len)
        y = pa.hstu_cand_fwd(*cargs, **ckw)
        for _ in range(2):
            pa.hstu_cand_fwd(*cargs, y=y, **ckw)
        torch.cuda.synchronize()
        print(json.dumps({"once": "cand", "workload": "mfalcon", "users": sp.batch,
                          "candidates": ci.total_cands}))
        return 0
    inp = hi.make_inputs(spec, seed=args.seed)
    d = lambda t: None if t is None else t.to("cuda").contiguous()
    q, k, v, u, offs = d(inp.q), d(inp.k), d(inp.v), d(inp.u), d(inp.offsets)
    kw = dict(timestamps=d(inp.timestamps), rab_pos=d(inp.rab_pos), rab_time=d(inp.rab_time),
              norm_len=inp.norm_len)
    bwd = args.once == "bwd"
    y, saved = pa.hstu_attn_fwd(q, k, v, u, offs, inp.max_seq_len, save_for_backward=bwd, **kw)
    for _ in range(2):
        if bwd:
            pa.hstu_attn_bwd(d(inp.dy), q, k, v, u, offs, inp.max_seq_len, saved, **kw)
        else:
            pa.hstu_attn_fwd(q, k, v, u, offs, inp.max_seq_len, y=y, **kw)
    torch.cuda.synchronize()
    print(json.dumps({"once": args.once, "workload": spec.name, "batch": spec.batch,
                      "tokens": inp.total_tokens}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="jagged", choices=sorted(hi.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--also", default="long,train,proj,mfalcon",
                    help="comma-separated workloads timed after the main one, 'proj' for the "
                         "projection GEMMs ('' for none)")
    ap.add_argument("--also-steps", type=int, default=50)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--cpu-budget-single", type=float, default=6.0)
    ap.add_argument("--ref-step-budget", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (profiling a smaller case)")
    ap.add_argument("--once", choices=["fwd", "bwd", "cand"], default=None,
                    help="run one forward, backward or candidate-scoring call twice and exit "
                         "(for ncu captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    spec = hi.WORKLOADS[args.workload]
    if args.batch > 0:
        if not args.once:
            ap.error("--batch only sizes the --once profiling runs")
        spec = hi.workload(args.workload, batch=args.batch)
    if args.once:
        return run_once(args, spec)
    if args.impl == "reference":
        return run_reference(args, spec)
    return run_gpu(args, spec)


if __name__ == "__main__":
    sys.exit(main())
