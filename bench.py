"""Benchmark of HSTU causal pointwise aggregated attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path over one batch of synthetic input:
for the forward workloads the fused attention + LayerNorm + gate forward, for
"train" the forward with saved statistics followed by the backward.  The
default workload is the model card's block shape ("neurarch": 8 sequences of
1024 tokens, 4 heads, d_qk = d_v = 128, position bias, bf16).

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
KERNEL_SOURCES = {
    "fwd": ["pointwise_attention_b200/csrc/fwd_sm100.cu", "pointwise_attention_b200/csrc/ptx.cuh",
            "pointwise_attention_b200/csrc/tile_math.cuh", "pointwise_attention_b200/csrc/internal.h"],
}


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


def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "%s.%s.txt" % (kernel_key, workload))
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    srcs = KERNEL_SOURCES.get("fwd")
    if fields.get("kernel_source_sha256") != source_digest(srcs):
        return None
    try:
        return int(float(fields["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed region."""

    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
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

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
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

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- oracle arm
def _row_sample(inp, stride: int):
    rows, fl = [], 0
    H, dqk, dv = inp.q.shape[1], inp.q.shape[2], inp.v.shape[2]
    for b, n in enumerate(inp.lengths):
        s = int(inp.offsets[b])
        for i in range(0, n, stride):
            rows.append(s + i)
            fl += 2 * (i + 1) * H * (dqk + dv)      # row i of a sequence: i+1 columns
    return rows, fl


def oracle_step_sample(inp, budget_s: float):
    """Times the oracle forward on the host cores: the whole workload if it fits
    in the budget, else every stride-th row (stride from a small probe); returns
    (flops, seconds, description)."""
    import numpy as np
    import oracle
    oracle.build()
    flops_full = hi.causal_flops(inp.lengths, inp.q.shape[1], inp.q.shape[2], inp.v.shape[2])
    probe_stride = max(1, int(math.ceil(flops_full / 2e9)))
    rows, fl = _row_sample(inp, probe_stride)
    t0 = time.perf_counter()
    oracle.fwd_rows(inp, np.array(rows, dtype=np.int64))
    rate = fl / max(time.perf_counter() - t0, 1e-9)
    if flops_full / rate <= budget_s:
        reps, total = 0, 0.0
        while reps == 0 or total < budget_s * 0.5:
            t0 = time.perf_counter()
            oracle.fwd(inp)
            total += time.perf_counter() - t0
            reps += 1
        return flops_full * reps, total, "full workload forward x%d" % reps
    stride = max(1, int(math.ceil(flops_full / rate / budget_s)))
    rows, fl = _row_sample(inp, stride)
    t0 = time.perf_counter()
    oracle.fwd_rows(inp, np.array(rows, dtype=np.int64))
    return fl, time.perf_counter() - t0, "every %d-th row of the workload (%d rows)" % (
        stride, len(rows))


def run_reference(args, spec):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = hi.make_inputs(spec, seed=args.seed)
    cores = os.cpu_count()
    for _ in range(args.warmup):
        oracle_step_sample(inp, budget_s=0.5)
    flops, secs = 0, 0.0
    desc = ""
    for _ in range(args.steps):
        f, s, desc = oracle_step_sample(inp, budget_s=args.ref_step_budget)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, **workload_config(spec)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm
def workload_config(spec):
    c = {"batch": spec.batch, "heads": spec.heads, "d_qk": spec.d_qk, "d_v": spec.d_v,
         "rab": "+".join(x for x, on in (("pos", spec.rab_pos_len > 0), ("time", spec.rab_time))
                         if on) or "none",
         "norm": "own_length" if spec.norm == "own" else "fixed"}
    if spec.len_range:
        c["seq_len"] = "U[%d,%d]" % spec.len_range
    else:
        c["seq_len"] = spec.seq_len
    return c


class Workload:
    """R device copies of one rank's inputs plus outputs and workspaces."""

    def __init__(self, inp, train: bool, device):
        import pointwise_attention_b200 as pa
        self.pa, self.inp, self.train = pa, inp, train
        per_set = algorithmic_bytes(inp)
        if train:
            per_set += inp.total_tokens * inp.q.shape[1] * inp.v.shape[2] * (4 + 2 * 5)
        self.R = max(2, int(math.ceil(2 * L2_BYTES / per_set)))
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
        self.launches_per_step = 1 if not train else 1 + 3   # forward; LN/gate, dQ, dK/dV backward kernels

    def step(self, i: int, stream=None):
        d, inp, pa = self.sets[i % self.R], self.inp, self.pa
        pa.hstu_attn_fwd(d["q"], d["k"], d["v"], d["u"], d["offsets"], inp.max_seq_len,
                         timestamps=d["ts"], rab_pos=d["rab_pos"], rab_time=d["rab_time"],
                         norm_len=inp.norm_len, save_for_backward=self.train, y=d["y"],
                         saved=d.get("saved"), workspace=d["ws"], stream=stream)
        if self.train:
            pa.hstu_attn_bwd(d["dy"], d["q"], d["k"], d["v"], d["u"], d["offsets"],
                             inp.max_seq_len, d["saved"], timestamps=d["ts"],
                             rab_pos=d["rab_pos"], rab_time=d["rab_time"],
                             norm_len=inp.norm_len, grads=d["grads"], workspace=d["ws"],
                             stream=stream)

    def backward(self, i: int, stream=None):
        d, inp, pa = self.sets[i % self.R], self.inp, self.pa
        pa.hstu_attn_bwd(d["dy"], d["q"], d["k"], d["v"], d["u"], d["offsets"],
                         inp.max_seq_len, d["saved"], timestamps=d["ts"],
                         rab_pos=d["rab_pos"], rab_time=d["rab_time"],
                         norm_len=inp.norm_len, grads=d["grads"], workspace=d["ws"],
                         stream=stream)

    def check(self):
        for d in self.sets:
            rc = self.pa.hstu_attn_check(d["ws"])
            if rc != 0:
                raise RuntimeError("device status after the timed region: %s"
                                   % self.pa.status_string(rc))


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

    inp = hi.make_inputs(spec, seed=rank_seed(args.seed, rank))
    train = spec.grad
    wl = Workload(inp, train, device)
    flops_fwd = hi.causal_flops(inp.lengths, spec.heads, spec.d_qk, spec.d_v)
    flops_step = flops_fwd * (1 + (2.5 if train else 0.0))

    for i in range(args.warmup):
        wl.step(i)
    torch.cuda.synchronize()
    wl.check()

    # CUDA graph of R consecutive steps (one per input set), replayed.
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        wl.step(0, stream=stream)           # warm the capture stream
        torch.cuda.current_stream().synchronize()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(wl.R):
                wl.step(i, stream=stream)
    torch.cuda.synchronize()
    reps, rest = divmod(args.steps, wl.R)
    tail = None
    if rest:
        tail = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(tail, stream=stream):
                for i in range(rest):
                    wl.step(i, stream=stream)
        torch.cuda.synchronize()
    for _ in range(2):                      # graph warm-up
        graph.replay()
    torch.cuda.synchronize()

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                graph.replay()
            if tail is not None:
                tail.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    elapsed = e0.elapsed_time(e1) / 1e3
    elapsed_max = reduce_max(elapsed, world, device)
    wl.check()

    value = flops_step * args.steps * world / elapsed_max / 1e12
    peaks, peak_kind = load_peaks()
    sec_per_step = elapsed / args.steps
    # Roofline of the dominant kernel (the forward for forward workloads).
    bytes_launch = algorithmic_bytes(inp)
    # One forward launch per step, replayed back to back from the graph: the
    # average launch duration is the timed region over the number of steps.
    t_launch = sec_per_step if not train else None
    roof = None
    if t_launch is not None:
        t_hbm = bytes_launch / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops_fwd / (peaks["bf16_tflops"] * 1e12)
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": bytes_launch / t_launch / 1e9,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        else:
            roof = {"bound": "tensor", "achieved": flops_fwd / t_launch / 1e12,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = profiled_traffic("hstu_fwd_bf16_sm100", spec.name)
        roof["peak_source"] = peak_kind + (" burst" if roof["bound"] == "tensor" else "")
        roof["kernel"] = "hstu_fwd_bf16_sm100" if spec.dtype == "bf16" else "fwd_simt<float>"
        roof["algorithmic_bytes"] = bytes_launch
        roof["algorithmic_flops"] = flops_fwd

    if train:
        # Training: the backward call (LN/gate, dQ and dK/dV kernels: two thirds
        # of the step in the ncu launch list) is the dominant unit.  It is timed
        # on its own: a graph of R backward calls, replayed, on the saved
        # outputs the timed steps left behind.
        bgraph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(bgraph, stream=stream):
                for i in range(wl.R):
                    wl.backward(i, stream=stream)
        torch.cuda.synchronize()
        for _ in range(2):
            bgraph.replay()
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        breps = max(1, reps)
        with torch.cuda.stream(stream):
            b0.record(stream)
            for _ in range(breps):
                bgraph.replay()
            b1.record(stream)
        torch.cuda.synchronize()
        t_bwd = b0.elapsed_time(b1) / 1e3 / (breps * wl.R)
        flops_bwd = 2.5 * flops_fwd
        roof = {"bound": "tensor", "achieved": flops_bwd / t_bwd / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = None
        roof["peak_source"] = peak_kind + " burst"
        roof["kernel"] = "hstu_attn_bwd (bwd_pre_simt, hstu_bwd_dq_sm100, hstu_bwd_dkdv_sm100)"
        roof["algorithmic_flops"] = flops_bwd
        roof["ms_per_call"] = t_bwd * 1e3
        wl.check()

    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    e2e_t, h2d, d2h = timed_e2e(wl, e2e_steps, device)
    e2e_t = reduce_max(e2e_t, world, device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, s, desc = oracle_step_sample(inp, budget_s=args.cpu_budget)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
               "kind": "oracle", "sample": desc}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    tensor_peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_max / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if spec.dtype == "bf16" else "f32", "data": "synthetic",
        "pct_of_dense_bf16_peak": 100.0 * value / world / tensor_peak,
        "config": {"workload": spec.name, **workload_config(spec),
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "%d rotating input sets (%.0f MB each) > 2x 126 MB L2" % (
                       wl.R, algorithmic_bytes(inp) / 1e6),
                   "timing": "CUDA graph of %d steps, CUDA events" % wl.R},
        "gpu_launches": args.steps * wl.launches_per_step,
        "roofline": roof,
        "cpu_baseline": cpu,
        "clocks": clk.summary(),
    }
    line["e2e"] = {"value": flops_step * world * e2e_steps / e2e_t / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "steps": e2e_steps}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="neurarch", choices=sorted(hi.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-step-budget", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    spec = hi.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, spec)
    return run_gpu(args, spec)


if __name__ == "__main__":
    sys.exit(main())
