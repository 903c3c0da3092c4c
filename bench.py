#!/usr/bin/env python
"""Benchmark of the MoE routing hot path (gate -> layout -> dispatch -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill] [--impl ours|reference]

One step = one pass of the four steps over one batch of the workload, with
inputs resident in HBM.  L2 is flushed (a write of twice its size) before every
step, outside the timed events.  Each op is bracketed by CUDA events on the
stream it runs on; ``value`` is whole-job tokens/s (all ranks' tokens over the
slowest rank's summed step time).  ``e2e`` repeats the measurement through the
same public API with pinned HOST inputs: the host->device copies of the step's
inputs and the device->host copy of its output are inside the timed region.

For N > 1 (torchrun, one process per GPU) every rank routes its own batch:
the work shards by tokens with no data-path collective ("weak" scaling); NCCL
is only used for the barrier and the max over ranks of the timed interval.

``--impl reference`` times the plain single-threaded CPU oracle on a bounded
sample of the same workload (rank 0 only), the comparison arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from combine_moe_topk_gate_b200.workloads import WORKLOADS, algorithmic_bytes, make_inputs  # noqa: E402

METRIC = "dispatch+combine tokens/s and effective HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = {
    "combine": "combine_moe_topk_gate_b200/csrc/combine.cu",
    "dispatch": "combine_moe_topk_gate_b200/csrc/dispatch.cu",
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="prefill", choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-backward", action="store_true",
                   help="skip timing the backward ops, the dispatch payload variants and the aligned layout")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the per-workload summary of the other four workloads")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle baseline CPU budget (s)")
    p.add_argument("--tokens", type=int, default=None,
                   help="override the workload's token count (profiling captures of a smaller case)")
    return p.parse_args()


def describe(w) -> str:
    gate = {"softmax": "softmax", "softmax_renorm": "softmax renormalised",
            "sigmoid_group": f"sigmoid group-limited ({w.n_groups} groups, top-{w.topk_groups} groups, "
                             f"group score = top-{w.group_topn} sum)"}[w.gate]
    return (f"{w.name}: N={w.N} tokens, H={w.H}, E={w.E} experts, top-{w.k}, {gate}, "
            f"R={w.R} logical ranks, {w.dtype.upper()} dispatch, BF16 combine, "
            f"expert outputs {'= dispatched rows' if w.expert_out == 'identity' else 'seeded bf16 N(0,1)'}")


def config_of(w, world: int) -> dict:
    """The workload description both arms print (ours and the oracle arm)."""
    return {"workload": describe(w), "tokens_per_gpu": w.N, "hidden": w.H, "experts": w.E,
            "topk": w.k, "logical_ranks": w.R, "payload": f"x bf16, dispatch {w.dtype}, out bf16",
            "l2": "flushed before every step, outside the events: a write of 2x the L2 size, "
                  "then a read of another 2x L2 buffer (the step starts cold and clean)",
            "timing": "step captured once as a CUDA graph and replayed; step time from events "
                      "at the graph's ends, per-op times from a second graph with event nodes "
                      "between the ops; medians over the timed steps",
            "parallelism": f"replicas x{world} (tokens sharded, no collective)"}


def host_description() -> dict:
    """Host cores and CPU model (the machine the oracle baseline runs on)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(op: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the capture (or there is none)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload][op]
        if e.get("source_sha256_16") != source_hash(KERNEL_SOURCES[op]):
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


def launches_per_step(w) -> int:
    """Kernels one step launches: routing (one launch when all N*k entries fit
    one 1024-entry chunk and E <= 512; else the gate and the layout's one or
    two launches), dispatch, combine."""
    small = w.N * w.k <= 1024
    route = 1 if small and w.E <= 512 else (2 if small else 3)
    return route + 1 + 1


def isolated_op_times(step_ops, flush, device, reps=30):
    """Each op alone in its own CUDA graph (cold, clean L2 before every replay);
    the empty graph's time is subtracted.  Inside the step an op can also pay for
    the previous op's dirty L2 lines, which this isolates."""
    ops = step_ops()
    out = {}
    for name in ["empty", *ops]:
        a = torch.cuda.Event(enable_timing=True, external=True)
        b = torch.cuda.Event(enable_timing=True, external=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            a.record(torch.cuda.current_stream(device))
            if name != "empty":
                ops[name]()
            b.record(torch.cuda.current_stream(device))
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            g.replay()
            b.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        ts.sort()
        out[name] = ts[len(ts) // 2]
    base = out.pop("empty")
    return {k: round(max(0.0, v - base), 2) for k, v in out.items()}


# ---------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's ``x`` (all ranks call this in the same order)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, world: int, steps: int, max_total_ms: float) -> float:
    """Tokens of all ranks over the slowest rank's timed interval, per second."""
    return tokens_per_rank * world * steps / (max_total_ms * 1e-3)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (read-only) for SM clock and clock-event reasons while running."""
    REASONS = {
        "gpu_idle": "nvmlClocksEventReasonGpuIdle",
        "applications_clocks_setting": "nvmlClocksEventReasonApplicationsClocksSetting",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "sync_boost": "nvmlClocksEventReasonSyncBoost",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.ok = period_s, False
        self._stop = threading.Event()
        try:
            import pynvml as N
            self.N = N
            N.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = None
            for i in range(N.nvmlDeviceGetCount()):
                h = N.nvmlDeviceGetHandleByIndex(i)
                u = N.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self.h = h
            if self.h is None:
                self.h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                mask = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if mask & getattr(N, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- reference arm
def oracle_step(w, inp, n):
    """One pass of the oracle over the first n tokens of the batch."""
    import numpy as np
    import oracle as O
    logits = inp.logits[:n].numpy()
    x = inp.x[:n].contiguous().view(torch.int16).numpy().view(np.uint16)
    idx, wts = O.topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    L = O.get_layout(idx, w.E, w.R)
    recv, _, _ = O.dispatch(x, L.token_slot, w.dtype_code)
    if w.expert_out == "identity":
        y = recv
    else:
        y = inp.y[: n * w.k].contiguous().view(torch.int16).numpy().view(np.uint16)
    O.combine(y, L.token_slot, wts)


def oracle_sample_size(w, inp, budget_s):
    n0 = min(w.N, 32)
    t = time.perf_counter()
    oracle_step(w, inp, n0)
    per_tok = (time.perf_counter() - t) / n0
    return max(1, min(w.N, int(budget_s / per_tok))), per_tok


def cpu_baseline(w, inp, budget_s):
    """Oracle passes over (a prefix of) the batch, repeated until budget_s of CPU work."""
    n, _ = oracle_sample_size(w, inp, budget_s)
    reps, t = 0, time.perf_counter()
    while True:
        oracle_step(w, inp, n)
        reps += 1
        dt = time.perf_counter() - t
        if dt >= budget_s:
            break
    return {"value": n * reps / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} pass(es) over the first {n} of the {w.N} tokens of the {w.name} batch "
                      f"(seed 0): gate+layout+dispatch+combine, single-threaded C oracle, {dt:.1f} s",
            **host_description()}


def workload(args):
    w = WORKLOADS[args.workload]
    return w if args.tokens is None else w.scaled(args.tokens)


def run_reference(args, rank, world):
    w = workload(args)
    if rank != 0:
        return
    inp = make_inputs(w, 0)
    budget = 60.0 / max(1, args.steps + args.warmup)
    n, per_tok = oracle_sample_size(w, inp, budget)
    for _ in range(args.warmup):
        oracle_step(w, inp, n)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, inp, n)
    dt = time.perf_counter() - t
    v = n * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_of(w, world),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: gate+layout+dispatch+combine over the first {n} of the "
                                   f"{w.N} tokens of the {w.name} batch (seed 0), single-threaded C oracle",
                         **host_description()},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
OPS = ("route", "dispatch", "combine")


class L2Flush:
    """Before every timed step: write a buffer of twice the L2 size (evicts
    every line), then read another one (so the lines left behind are clean,
    not dirty lines the next step would have to write back)."""

    def __init__(self, device):
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        self.w = torch.empty(2 * l2, dtype=torch.uint8, device=device)
        self.r = torch.zeros(2 * l2 // 4, dtype=torch.float32, device=device)

    def zero_(self):
        self.w.zero_()
        self.r.max()


class StepRunner:
    """Device buffers of one workload and the four calls of one step, each
    through the library's public binding."""

    def __init__(self, api, w, inp, device):
        self.api, self.w, self.device = api, w, device
        self.logits = inp.logits.to(device)
        self.x = inp.x.to(device)
        self.y_in = inp.y.to(device) if inp.y is not None else None
        self.idx = torch.empty((w.N, w.k), dtype=torch.int32, device=device)
        self.wts = torch.empty((w.N, w.k), dtype=torch.float32, device=device)
        self.L = api.Layout.empty(w.N, w.k, w.E, w.R, device, route=True)
        # the same two steps as separate calls (timed alone, for the breakdown)
        self.idx2 = torch.empty_like(self.idx)
        self.wts2 = torch.empty_like(self.wts)
        self.L2 = api.Layout.empty(w.N, w.k, w.E, w.R, device)
        if w.dtype != "bf16":
            self.recv = torch.empty((w.S, w.H), dtype=torch.uint8, device=device)
            shape, sdt = api.scale_shape(w.S, w.H, w.dtype_code)
            self.scale = torch.empty(shape, dtype=sdt, device=device)
        else:
            self.recv = torch.empty((w.S, w.H), dtype=torch.bfloat16, device=device)
            self.scale = None
        self.out = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=device)
        self.y = self.recv if w.expert_out == "identity" else self.y_in

    def ops(self, stream=None):
        """The step: gate and layout in one call (moe_route, which also has L2
        fetch x for the dispatch that follows), dispatch, combine."""
        api, w, L = self.api, self.w, self.L
        return {
            "route": lambda: api.moe_route(self.logits, w.k, w.gate_kind, w.n_groups, w.topk_groups,
                                           w.group_topn, w.R, topk_idx=self.idx, topk_w=self.wts, out=L,
                                           prefetch=self.x, stream=stream),
            "dispatch": lambda: api.moe_dispatch(self.x, L.token_slot, w.dtype_code, recv_x=self.recv,
                                                 recv_scale=self.scale, d_status=L.status, stream=stream),
            "combine": lambda: api.moe_combine(self.y, L.token_slot, self.wts, out=self.out,
                                               d_status=L.status, stream=stream),
        }

    def separate_ops(self, stream=None):
        """Gate and layout as the two separate calls."""
        api, w = self.api, self.w
        return {
            "gate": lambda: api.moe_topk_gate(self.logits, w.k, w.gate_kind, w.n_groups, w.topk_groups,
                                              w.group_topn, topk_idx=self.idx2, topk_w=self.wts2, stream=stream),
            "layout": lambda: api.moe_get_layout(self.idx2, w.E, w.R, out=self.L2, stream=stream),
        }

    def step(self, ev=None):
        stream = torch.cuda.current_stream(self.device)  # the capture stream inside torch.cuda.graph
        for j, fn in enumerate(self.ops(stream).values()):
            if ev:
                ev[j].record(stream)
            fn()
        if ev:
            ev[len(OPS)].record(stream)

    def check_status(self, when: str):
        if int(self.L.status.item()) != 0:
            raise RuntimeError(f"device status {int(self.L.status.item())} {when}")

    def capture(self, flush, warmup: int):
        """Eager warm-up, then the step captured once as a CUDA graph and
        replayed, so the timed interval is device time of the kernels back to
        back (their launches overlap through programmatic dependent launch),
        not the binding's launch overhead.  graph_step has events only at its
        ends and gives the step time; graph_ops has an event-record node
        between the ops (which also cuts the launch overlap) and gives the
        per-op breakdown."""
        for _ in range(warmup):
            flush.zero_()
            self.step()
        torch.cuda.synchronize(self.device)
        self.check_status("after warm-up")
        dev = self.device
        self.ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        self.graph_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_step):
            self.ends[0].record(torch.cuda.current_stream(dev))
            self.step()
            self.ends[1].record(torch.cuda.current_stream(dev))
        self.evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(OPS) + 1)]
        self.graph_ops = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_ops):
            self.step(self.evs)
        for _ in range(warmup):
            for g in (self.graph_step, self.graph_ops):
                flush.zero_()
                g.replay()
        torch.cuda.synchronize(dev)

    def timed(self, steps: int, flush):
        """(step times in ms, {op: [ms]}) over `steps` replays of each graph."""
        step_ms, per_op = [], {n: [] for n in OPS}
        for _ in range(steps):
            flush.zero_()
            self.graph_step.replay()
            self.ends[1].synchronize()
            step_ms.append(self.ends[0].elapsed_time(self.ends[1]))
        for _ in range(steps):
            flush.zero_()
            self.graph_ops.replay()
            self.evs[-1].synchronize()
            for j, n in enumerate(OPS):
                per_op[n].append(self.evs[j].elapsed_time(self.evs[j + 1]))
        torch.cuda.synchronize(self.device)
        self.check_status("after the timed steps")
        return step_ms, per_op


def summary_of(w, step_ms, per_op, isolated, peak, world=1) -> dict:
    """Medians of one workload's timed steps, with the dispatch and combine
    roofline fractions (in the step and alone).  Decode- and tiny-sized steps
    move a few MB and are bound by launch and memory latency, not bandwidth:
    their fractions are reported but do not describe the kernels' bound."""
    ab = algorithmic_bytes(w)
    ab["route"] = ab["gate"] + ab["layout"]
    med = {n: statistics.median(v) * 1e3 for n, v in per_op.items()}
    st = statistics.median(step_ms) * 1e3
    latency_bound = ab["combine"] < 64e6
    ops = {}
    for n in ("dispatch", "combine"):
        iso = isolated.get(n) or None
        ops[n] = {"in_step_us": round(med[n], 2), "frac": ab[n] / (med[n] * 1e-6) / 1e9 / peak,
                  "isolated_us": iso, "isolated_frac": (ab[n] / (iso * 1e-6) / 1e9 / peak) if iso else None,
                  "algorithmic_bytes": ab[n]}
    return {"config": describe(w), "tokens": w.N,
            "step_us": {"median": round(st, 2), "mean": round(statistics.mean(step_ms) * 1e3, 2),
                        "min": round(min(step_ms) * 1e3, 2), "max": round(max(step_ms) * 1e3, 2)},
            "tokens_per_s": w.N * world / (st * 1e-6),
            "per_op_us": {n: round(v, 2) for n, v in med.items()},
            "per_op_us_mean": {n: round(statistics.mean(v) * 1e3, 2) for n, v in per_op.items()},
            "isolated_us": isolated,
            "dispatch_combine_tokens_per_s": w.N * world / ((med["dispatch"] + med["combine"]) * 1e-6),
            **ops, "bound": "latency" if latency_bound else "hbm"}


def other_workloads(api, main, device, steps, warmup, flush, peak) -> dict:
    """Every other workload measured the same way (seed 0), one after another."""
    res = {}
    for name in ("tiny", "decode", "prefill", "skewed", "mixtral"):
        if name == main:
            continue
        w = WORKLOADS[name]
        r = StepRunner(api, w, make_inputs(w, 0), device)
        r.capture(flush, warmup)
        step_ms, per_op = r.timed(steps, flush)
        iso = isolated_op_times(r.ops, flush, device)
        iso.update(isolated_op_times(r.separate_ops, flush, device))
        res[name] = summary_of(w, step_ms, per_op, iso, peak)
        res[name]["quant_fp8_channel"] = channel_fp8_time(api, r, flush, device, peak)
        if name in ("mixtral", "skewed"):   # top-2 / H = 4096 and the skewed top-8 shape
            api.moe_route(r.logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn, w.R,
                          topk_idx=r.idx, topk_w=r.wts, out=r.L)
            res[name]["dispatch_variants"] = dispatch_variant_times(api, w, r.x, r.L, flush, device)
        del r
        torch.cuda.empty_cache()
    return res


def dispatch_variant_times(api, w, x, L, flush, device) -> dict:
    """Every dispatch payload type on this batch's layout, each alone (cold,
    clean L2): µs, fraction of the measured copy peak, algorithmic bytes."""
    from combine_moe_topk_gate_b200.workloads import DTYPES, Workload
    bufs = {}
    for dname, code in DTYPES.items():
        rx = torch.empty((w.S, w.H), dtype=torch.bfloat16 if code == 0 else torch.uint8, device=device)
        shape, sdt = api.scale_shape(w.S, w.H, code)
        bufs[dname] = (code, rx, torch.empty(shape, dtype=sdt, device=device) if shape else None)
    nv = None
    if w.H % 64 == 0:
        nv = (torch.empty((w.S, w.H // 2), dtype=torch.uint8, device=device),
              torch.empty((w.S, w.H // 16), dtype=torch.uint8, device=device),
              torch.empty((w.S,), dtype=torch.float32, device=device))
    e5 = torch.empty((w.S, w.H // 2 * 3), dtype=torch.uint8, device=device) if w.H % 32 == 0 else None
    tiled = None
    if w.H % 128 == 0:   # MXFP8 with the block-scaled MMA's tiled E8M0 scales
        shape_t, sdt_t = api.scale_shape(w.S, w.H, api.MOE_DTYPE_MXFP8_E4M3, api.MOE_SCALE_MMA_TILED)
        if shape_t:
            tiled = (torch.empty((w.S, w.H), dtype=torch.uint8, device=device),
                     torch.empty(shape_t, dtype=sdt_t, device=device))

    def var_ops():
        ops = {d: (lambda c=c, rx=rx, rs=rs: api.moe_dispatch(x, L.token_slot, c, recv_x=rx, recv_scale=rs,
                                                             d_status=L.status))
               for d, (c, rx, rs) in bufs.items()}
        if nv is not None:
            ops["nvfp4"] = lambda: api.moe_dispatch_nvfp4(x, L.token_slot, recv_x=nv[0], block_scale=nv[1],
                                                          row_scale=nv[2], d_status=L.status)
        if e5 is not None:
            ops["e5m6"] = lambda: api.moe_dispatch(x, L.token_slot, api.MOE_DTYPE_E5M6, recv_x=e5,
                                                   d_status=L.status)
        if tiled is not None:
            ops["mxfp8_mma_tiled"] = lambda: api.moe_dispatch(
                x, L.token_slot, api.MOE_DTYPE_MXFP8_E4M3, recv_x=tiled[0], recv_scale=tiled[1],
                scale_layout=api.MOE_SCALE_MMA_TILED, d_status=L.status)
        return ops
    vt = isolated_op_times(var_ops, flush, device)
    peak_v, _ = measured_peak()
    variants = {}
    for d, us in vt.items():
        abv = algorithmic_bytes(Workload(**{**w.__dict__, "dtype": "mxfp8" if d == "mxfp8_mma_tiled" else d}))
        abv = abv["dispatch"]
        variants[d] = {"us": us, "frac": abv / (us * 1e-6) / 1e9 / peak_v if us else None,
                       "algorithmic_bytes": abv}
    torch.cuda.synchronize(device)
    if int(L.status.item()) != 0:
        raise RuntimeError(f"device status {int(L.status.item())} after the dispatch variants")
    return variants


def channel_fp8_time(api, r, flush, device, peak, align: int = 128) -> dict:
    """Per-(expert, channel) FP8 of a seeded bf16 receive buffer laid out by
    this batch's GEMM-aligned layout (the weight-gradient GEMM's operand),
    alone with a clean cold L2; bytes = the landed rows read once and their
    codes written once, plus the scales."""
    w = r.w
    api.moe_route(r.logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn, w.R,
                  topk_idx=r.idx, topk_w=r.wts, out=r.L)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    La = api.Layout.empty(w.N, w.k, w.E, w.R, device, align=align)
    api.moe_get_layout(r.idx, w.E, w.R, align=align, out=La)
    y = torch.empty((rows, w.H), dtype=torch.bfloat16, device=device).normal_(generator=torch.Generator(
        device=device).manual_seed(11))
    out = torch.empty((rows, w.H), dtype=torch.uint8, device=device)
    sc = torch.empty((w.E, w.H), dtype=torch.float32, device=device)
    ws = torch.zeros(api.moe_quant_fp8_channel_workspace_bytes(w.E, w.H), dtype=torch.uint8, device=device)
    us = isolated_op_times(lambda: {"quant_fp8_channel": lambda: api.moe_quant_fp8_channel(
        y, La.expert_offset, La.expert_count, out=out, scale=sc, workspace=ws, d_status=La.status)}, flush,
        device)
    us = us["quant_fp8_channel"]
    counts = La.expert_count.cpu()
    landed = int(counts.sum().item())
    nbytes = landed * w.H * 3 + 4 * w.E * w.H + 8 * w.E
    torch.cuda.synchronize(device)
    if int(La.status.item()) != 0:
        raise RuntimeError(f"device status {int(La.status.item())} after the per-channel FP8")
    return {"us": us, "frac": nbytes / (us * 1e-6) / 1e9 / peak if us else None, "algorithmic_bytes": nbytes,
            "landed_rows": landed, "max_expert_rows": int(counts.max().item()),
            "mean_expert_rows": landed / w.E}


def run_ours(args, rank, world, device):
    from combine_moe_topk_gate_b200 import api
    w = workload(args)
    inp = make_inputs(w, rank)
    stream = torch.cuda.current_stream(device)
    flush = L2Flush(device)
    r = StepRunner(api, w, inp, device)
    r.capture(flush, args.warmup)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clk:
        step_ms, per_op = r.timed(args.steps, flush)
        if world > 1:
            torch.distributed.barrier()
        max_total_ms = max_over_ranks(sum(step_ms), world, device)

        isolated = isolated_op_times(r.ops, flush, device)
        isolated.update(isolated_op_times(r.separate_ops, flush, device))
        L, idx, wts, x, y_in, out = r.L2, r.idx, r.wts, r.x, r.y_in, r.out
        api.moe_get_layout(idx, w.E, w.R, out=L)   # the separate-call handle, for the sections below
        recv = r.recv
        peak, peak_kind = measured_peak()
        workloads = None
        if world == 1 and not args.no_workloads and args.tokens is None:
            workloads = {w.name: summary_of(w, step_ms, per_op, isolated, peak)}
            workloads[w.name]["quant_fp8_channel"] = channel_fp8_time(api, r, flush, device, peak)
            workloads.update(other_workloads(api, w.name, device, args.steps, args.warmup, flush, peak))
        backward = None
        if not args.no_backward:
            # backward ops on the same layout, timed alone (cold, clean L2)
            gen = torch.Generator(device="cpu").manual_seed(1234)
            grad_recv = torch.randn(w.S, w.H, generator=gen).to(torch.bfloat16).to(device)
            grad_out = torch.randn(w.N, w.H, generator=gen).to(torch.bfloat16).to(device)
            y_b = y_in if y_in is not None else torch.randn(w.S, w.H, generator=gen).to(torch.bfloat16).to(device)
            grad_x = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=device)
            grad_y = torch.empty((w.S, w.H), dtype=torch.bfloat16, device=device)
            grad_w = torch.empty((w.N, w.k), dtype=torch.float32, device=device)

            def bwd_ops():
                return {
                    "dispatch_backward": lambda: api.moe_dispatch_backward(
                        grad_recv, L.token_slot, grad_x=grad_x, d_status=L.status),
                    "combine_backward": lambda: api.moe_combine_backward(
                        grad_out, y_b, L.token_slot, wts, grad_y=grad_y, grad_w=grad_w, d_status=L.status),
                }
            bt = isolated_op_times(bwd_ops, flush, device)
            ab_all = algorithmic_bytes(w)
            peak_b, _ = measured_peak()
            backward = {n: {"us": bt[n], "gbs": ab_all[n] / (bt[n] * 1e-6) / 1e9 if bt[n] else None,
                            "frac": ab_all[n] / (bt[n] * 1e-6) / 1e9 / peak_b if bt[n] else None,
                            "algorithmic_bytes": ab_all[n]} for n in bt}
            torch.cuda.synchronize(device)
            if int(L.status.item()) != 0:
                raise RuntimeError(f"device status {int(L.status.item())} after the backward ops")

        variants = None
        if not args.no_backward:
            variants = dispatch_variant_times(api, w, x, L, flush, device)

        aligned = None
        if not args.no_backward:
            # the GEMM-aligned layout (every expert's rows start at a multiple of
            # 128, one M tile) and the ops on its padded buffer, each alone
            from combine_moe_topk_gate_b200.workloads import Workload
            A = 128
            rows_a = api.moe_aligned_recv_rows(w.N, w.k, w.E, A)
            La = api.Layout.empty(w.N, w.k, w.E, w.R, device, align=A)
            api.moe_get_layout(idx, w.E, w.R, align=A, out=La)
            rx_a = torch.empty((rows_a, w.H), dtype=recv.dtype, device=device)
            shape_a, sdt_a = api.scale_shape(rows_a, w.H, w.dtype_code)
            rs_a = torch.empty(shape_a, dtype=sdt_a, device=device) if shape_a else None
            y_a = torch.empty((rows_a, w.H), dtype=torch.bfloat16, device=device).normal_()
            out_a = torch.empty_like(out)

            # the same rows with the scales laid out for the grouped GEMM: MN-major
            # (per-block FP8) and the block-scaled MMA's tiled E8M0 atoms (MXFP8)
            gemm_scales = {}
            if w.H % 128 == 0:
                rx8 = torch.empty((rows_a, w.H), dtype=torch.uint8, device=device)
                for nm, dt, lay in (("dispatch_fp8_mn_major", api.MOE_DTYPE_FP8_E4M3, api.MOE_SCALE_MN_MAJOR),
                                    ("dispatch_mxfp8_mma_tiled", api.MOE_DTYPE_MXFP8_E4M3, api.MOE_SCALE_MMA_TILED)):
                    shp, sdt = api.scale_shape(rows_a, w.H, dt, lay)
                    gemm_scales[nm] = (dt, lay, torch.empty(shp, dtype=sdt, device=device))

            # SwiGLU + FP8 quantisation between the expert GEMMs, on the same padded
            # rows: h = [gate | up] of the first GEMM (seeded, resident), I = the
            # experts' intermediate width (2048 for the 7168-wide configs, 14336
            # for Mixtral 8x7B)
            inter = 14336 if w.name == "mixtral" else 2048
            h_a = torch.empty((rows_a, 2 * inter), dtype=torch.bfloat16, device=device).normal_()
            sw_out = torch.empty((rows_a, inter), dtype=torch.uint8, device=device)
            shp, sdt = api.scale_shape(rows_a, inter, api.MOE_DTYPE_FP8_E4M3, api.MOE_SCALE_MN_MAJOR)
            sw_sc = torch.empty(shp, dtype=sdt, device=device)

            # per-(expert, channel) FP8 of a bf16 receive buffer (the weight-gradient
            # GEMM's operand); y_a doubles as that buffer
            ch_out = torch.empty((rows_a, w.H), dtype=torch.uint8, device=device)
            ch_sc = torch.empty((w.E, w.H), dtype=torch.float32, device=device)
            ch_ws = torch.zeros(api.moe_quant_fp8_channel_workspace_bytes(w.E, w.H), dtype=torch.uint8,
                                device=device)

            def al_ops():
                ops = {
                    "quant_fp8_channel": lambda: api.moe_quant_fp8_channel(
                        y_a, La.expert_offset, La.expert_count, out=ch_out, scale=ch_sc, workspace=ch_ws,
                        d_status=La.status),
                    "swiglu_fp8_mn_major": lambda: api.moe_swiglu_quant(
                        h_a, api.MOE_DTYPE_FP8_E4M3, slot_token=La.slot_token, scale_layout=api.MOE_SCALE_MN_MAJOR,
                        out=sw_out, out_scale=sw_sc),
                    "layout": lambda: api.moe_get_layout(idx, w.E, w.R, align=A, out=La),
                    "dispatch": lambda: api.moe_dispatch(x, La.token_slot, w.dtype_code, recv_x=rx_a,
                                                         recv_scale=rs_a, d_status=La.status),
                    "combine": lambda: api.moe_combine(y_a, La.token_slot, wts, out=out_a, d_status=La.status),
                }
                for nm, (dt, lay, buf) in gemm_scales.items():
                    ops[nm] = (lambda dt=dt, lay=lay, buf=buf: api.moe_dispatch(
                        x, La.token_slot, dt, recv_x=rx8, recv_scale=buf, scale_layout=lay, d_status=La.status))
                return ops
            at = isolated_op_times(al_ops, flush, device)
            torch.cuda.synchronize(device)
            if int(La.status.item()) != 0:
                raise RuntimeError(f"device status {int(La.status.item())} after the aligned ops")
            peak_a, _ = measured_peak()
            ab_a = algorithmic_bytes(w)
            landed = int((La.slot_token >= 0).sum().item())
            ab_a["quant_fp8_channel"] = landed * w.H * 3 + 4 * w.E * w.H + 8 * w.E
            ab_a["swiglu_fp8_mn_major"] = landed * (4 * inter + inter + 4 * (inter // 128)) + 4 * rows_a
            ab_a["dispatch_fp8_mn_major"] = algorithmic_bytes(Workload(**{**w.__dict__, "dtype": "fp8"}))["dispatch"]
            ab_a["dispatch_mxfp8_mma_tiled"] = algorithmic_bytes(Workload(**{**w.__dict__, "dtype": "mxfp8"}))["dispatch"]
            aligned = {"align": A, "recv_rows": rows_a,
                       "padding_rows": int(rows_a - w.S), "swiglu_inter": inter, "landed_rows": landed,
                       **{n: {"us": us, "frac": (ab_a[n] / (us * 1e-6) / 1e9 / peak_a)
                              if us and n != "layout" else None}
                          for n, us in at.items()}}
            del rx_a, rs_a, y_a, La, gemm_scales, h_a, sw_out, sw_sc, ch_out, ch_sc

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, w, inp, device, stream, r.step, r.logits, r.x, r.y_in, r.out, flush, world)

    if rank != 0:
        return
    ab = algorithmic_bytes(w)
    ab["route"] = ab["gate"] + ab["layout"]
    med = {n: statistics.median(v) for n, v in per_op.items()}
    gbs = {n: ab[n] / (med[n] * 1e-3) / 1e9 for n in med}
    dominant = max(("dispatch", "combine"), key=lambda n: med[n])
    other = "dispatch" if dominant == "combine" else "combine"

    def roof(n):
        iso = isolated.get(n) or None
        return {"kernel": n, "bound": "hbm", "achieved": gbs[n], "peak": peak, "unit": "GB/s",
                "frac": gbs[n] / peak, "peak_source": f"{peak_kind} hbm_gbs",
                "traffic": ncu_traffic(n, w.name), "algorithmic_bytes": ab[n],
                "median_launch_us": 1e3 * med[n],
                "isolated_us": iso,
                "isolated_frac": (ab[n] / (iso * 1e-6) / 1e9 / peak) if iso else None}

    line = {
        "impl": "ours", "metric": METRIC,
        "value": whole_job_rate(w.N, world, args.steps, max_total_ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": max_total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(w, world),
        "step_us_median": statistics.median(step_ms) * 1e3,
        "per_op_us": {n: 1e3 * v for n, v in med.items()},
        "per_op_gbs": gbs,
        "dispatch_combine_tokens_per_s": w.N * world / ((med["dispatch"] + med["combine"]) * 1e-3),
        "roofline": roof(dominant),
        "roofline_other": roof(other),
        "gpu_launches": 2 * launches_per_step(w) * args.steps,  # the two timed loops of the main workload
        "isolated_us": isolated,
        "workloads": workloads,
        "backward": backward,
        "dispatch_variants": variants,
        "aligned_layout": aligned,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, make_inputs(w, 0), args.cpu_seconds)
    print(json.dumps(line), flush=True)


def measure_e2e(args, w, inp, device, stream, step, logits, x, y_in, out, flush, world):
    """Same step through the public API with the inputs in pinned host memory."""
    h_logits = inp.logits.pin_memory()
    h_x = inp.x.pin_memory()
    h_y = inp.y.pin_memory() if inp.y is not None else None
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = h_logits.numel() * 4 + h_x.numel() * 2 + (h_y.numel() * 2 if h_y is not None else 0)
    d2h = h_out.numel() * 2

    def e2e_step():
        logits.copy_(h_logits, non_blocking=True)
        x.copy_(h_x, non_blocking=True)
        if h_y is not None:
            y_in.copy_(h_y, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)

    steps = max(3, min(args.steps, 20))
    for _ in range(3):
        flush.zero_()
        e2e_step()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    total = 0.0
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        total += a.elapsed_time(b)
    return {"value": whole_job_rate(w.N, world, steps, max_over_ranks(total, world, device)),
            "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
