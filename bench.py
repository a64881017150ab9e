"""Benchmark of the MoonEP hot path on B200.

One step = one pass of the whole path over one batch of the large training
shape (R=32 simulated ranks, E=384, K=8, S=4096, H=7168, B=12, Zipf-biased
routing at maxvio 1): plan -> dispatch -> combine -> combine backward ->
replica-gradient reduce (gate+up+down, 3*7168*2048 fp32 per expert).

Printed value (rank 0, one JSON line): dispatch+combine HBM GB/s, i.e. the
algorithmic bytes of the dispatch and combine launches of all ranks divided
by their CUDA-event time (max over ranks).  The planner's microseconds, every
kernel's roofline fraction, the maxvio sweep, an end-to-end number through
the public API with host buffers, and the CPU oracle's number on a bounded
sample are reported beside it.

--impl reference times the CPU oracle on the host cores instead (bounded
sample of the same workload per step), rank 0 only.

Multi-GPU: the simulated ranks already live on one GPU, so N GPUs run N
independent replicas of the step (weak scaling, no data-path collective);
NCCL is used only for the barrier and the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from load_balancing_moonep_b200 import workloads as W  # noqa: E402

METRIC = "dispatch+combine HBM GB/s (% of ~8 TB/s) vs maxvio; planner µs/layer"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------ byte models

def bytes_dispatch(wl) -> int:
    """read each token row once, write it K times, read dst_pos"""
    return wl.tokens * wl.H * 2 * (1 + wl.K) + wl.pairs * 4


def bytes_combine(wl) -> int:
    """read K rows per token, write one row, read dst_pos and w"""
    return wl.tokens * wl.H * 2 * (wl.K + 1) + wl.pairs * 8


def bytes_combine_bwd(wl) -> int:
    """read dy and K y rows, write K dy_buf rows; read dst_pos, w; write dw"""
    return wl.tokens * wl.H * 2 * (1 + 2 * wl.K) + wl.pairs * 12


def bytes_reduce(n_rep_prefetched: int, n_rep_experts: int, P: int) -> int:
    """each replica row read + zeroed, each home row read + written"""
    return (n_rep_prefetched + n_rep_experts) * P * 4 * 2


def bytes_prefetch(n_rep_prefetched: int, n_rep_experts: int, P: int, wl) -> int:
    """each expert with prefetched replicas read once, each replica's pool
    row written once (bf16), the slot table read and the weight-row table
    written"""
    return (n_rep_experts + n_rep_prefetched) * P * 2 + wl.R * wl.E * 8


def bytes_plan(wl) -> int:
    """two passes over the ids, dst_pos and row_src written"""
    return wl.pairs * 4 * 2 + wl.pairs * 4 * 2


# ------------------------------------------------------------------ peaks

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the source files each measured kernel is compiled from: a kernel's ncu
# counters stay valid while these are unchanged (the ABI header holds only
# declarations and constants and is left out)
KERNEL_SOURCES = {
    "dispatch": ("data.cu", "common.cuh"),
    "combine": ("data.cu", "common.cuh"),
    "combine_bwd": ("data.cu", "common.cuh"),
    "reduce": ("reduce.cu", "common.cuh"),
    "prefetch": ("prefetch.cu", "common.cuh"),
}


def kernel_sources_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "load_balancing_moonep_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic_ratio():
    """DRAM traffic / algorithmic bytes per launch, from the committed ncu
    summary of the reduced-size profile cases (``bench.py --profile KERNEL``),
    for each kernel whose sources are unchanged since the capture.  The
    per-launch traffic of a timed launch is this ratio times its algorithmic
    bytes: the per-token (per-row) bytes of these kernels do not depend on
    the number of tokens (rows), so traffic scales with the units processed."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return {}
    d = json.load(open(p))
    out = {}
    for k, v in d.get("kernels", {}).items():
        if k in KERNEL_SOURCES and v.get("sources_sha") == kernel_sources_hash(k):
            out[k] = v["dram_bytes_per_launch"] / v["alg_bytes_per_launch"]
    return out


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout: float = 3.0):
        """Until nvidia-smi has printed a sample: its start-up (driver and
        NVML initialisation) then lies outside the timed region."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def smi_index(local: int) -> str:
    """nvidia-smi's id for this process's GPU (CUDA_VISIBLE_DEVICES aware)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


# ------------------------------------------------------------ distributed

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        log(f"warning: --gpus {n_gpus} but WORLD_SIZE={world}; using WORLD_SIZE")
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


# A device-side sleep of about 50 us before a plan timed alone: the host
# enqueues the plan meanwhile, so its CUDA events time the device.
SPACER_CYCLES = 100_000


def count_library_launches(fn):
    """Kernels of this library one call of fn launches (a profiler trace of
    one untimed step): (count, how), or (None, reason)."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        n = sum(1 for e in prof.events()
                if e.device_type == torch.autograd.DeviceType.CUDA and "moonep::" in e.name)
        return n, "profiler trace of one untimed step: kernels named moonep::"
    except Exception as exc:  # profiler unavailable
        return None, f"no profiler trace: {type(exc).__name__}: {str(exc)[:120]}"


def max_over_ranks(world, x: float) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(world, x: float) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------ CPU oracle

def oracle_sample(wl, topk_np, w_np, hidden_sample_bits, tokens, y_rows_bits, lib=None, plan=True):
    """Time the CPU oracle on a bounded sample: the plan over the whole
    routing (unless plan=False), dispatch and combine over the sampled
    tokens (lib: the oracle build to run them with; default the
    single-threaded oracle).  Returns (plan_s, data_s, data_bytes)."""
    import oracle
    ocfg = oracle.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    t0 = time.perf_counter()
    info = oracle.plan(ocfg, topk_np)["info"] if plan else np.zeros(16, np.int32)
    t1 = time.perf_counter()
    n = len(tokens)
    sub = {"dst_pos": np.arange(n * wl.K, dtype=np.int32).reshape(n, wl.K), "info": info}
    scfg = oracle.Config(R=1, E=wl.E, K=wl.K, S=n, H=wl.H, B=0)
    buf = np.zeros((n * wl.K, wl.H), np.uint16)
    wsub = np.ascontiguousarray(w_np[tokens])
    t2 = time.perf_counter()
    oracle.dispatch(scfg, sub, hidden_sample_bits, buf, lib=lib)
    oracle.combine(scfg, sub, y_rows_bits, wsub, lib=lib)
    t3 = time.perf_counter()
    frac = n / wl.tokens
    data_bytes = (bytes_dispatch(wl) + bytes_combine(wl)) * frac
    return t1 - t0, t3 - t2, data_bytes


def oracle_reduce_sample(wl, topk_np, P, lib=None):
    """Time the oracle's replica-gradient reduce over the real plan on rows
    of P elements (a bounded sample of the gate+up+down rows).  Returns
    (seconds, algorithmic bytes)."""
    import oracle
    ocfg = oracle.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    op = oracle.plan(ocfg, topk_np)
    inf = oracle.info_dict(op)
    rng = np.random.default_rng(4)
    rb = rng.standard_normal((wl.R, wl.B, P), dtype=np.float32)
    hg = rng.standard_normal((wl.E, P), dtype=np.float32)
    t0 = time.perf_counter()
    oracle.reduce_replica_grads(ocfg, op, rb, hg, P, lib=lib)
    dt = time.perf_counter() - t0
    return dt, bytes_reduce(inf["n_rep"] - inf["n_overflow"], inf["n_rep_experts"], P)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sample_tokens(wl, n):
    return np.arange(min(n, wl.tokens), dtype=np.int64)


def cpu_inputs(wl, maxvio, n_tokens, device):
    r = W.routing(wl, maxvio, seed=0, device=device)
    topk = r.topk_idx.cpu().numpy()
    w = r.weights.cpu().numpy()
    tokens = sample_tokens(wl, n_tokens)
    hid = W.bits(W.bf16_normal((len(tokens), wl.H), seed=1, device="cpu"))
    y = W.bits(W.bf16_normal((len(tokens) * wl.K, wl.H), seed=2, device="cpu"))
    return r, topk, w, tokens, hid, y


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    r, topk, w, tokens, hid, y = cpu_inputs(wl, args.maxvio, args.ref_tokens, dev)
    times, plan_s = [], []
    for i in range(args.warmup + args.steps):
        ps, ds, db = oracle_sample(wl, topk, w, hid, tokens, y)
        if i >= args.warmup:
            times.append(ds)
            plan_s.append(ps)
    data_s = sum(times)
    value = db * len(times) / data_s / 1e9
    ms_step = (sum(times) + sum(plan_s)) / len(times) * 1e3
    sample = (f"per step: plan over all {wl.pairs} pairs + dispatch and combine of the first "
              f"{len(tokens)} of {wl.tokens} tokens, single-threaded C oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(wl, r, args),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cores": host_cores()},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "planner_us": round(statistics.median(plan_s) * 1e6, 1),
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, r, args):
    return {"workload": f"{wl.name}: R={wl.R} E={wl.E} K={wl.K} S={wl.S} H={wl.H} B={wl.B}",
            "R": wl.R, "E": wl.E, "K": wl.K, "S": wl.S, "H": wl.H, "B": wl.B,
            "maxvio_target": args.maxvio, "maxvio": round(r.maxvio, 4),
            "routing": f"gaussian logits + Zipf(s={wl.zipf_s}) expert bias, top-{wl.K}, seed 0",
            "l2": "inputs larger than L2 (hidden 1.9 GB, buffers 15 GB, 126 MB L2); no flush",
            "parallelism": "replicas (R ranks simulated in one GPU's HBM)"}


# ------------------------------------------------------------- our arm

class Timer:
    """CUDA events on the current stream around each call of a step."""

    def __init__(self):
        self.pairs = {}

    def mark(self, name):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        self.pairs.setdefault(name, []).append((s, e))
        s.record()
        return e

    def total_ms(self, name):
        return sum(s.elapsed_time(e) for s, e in self.pairs.get(name, []))

    def times_ms(self, name):
        return [s.elapsed_time(e) for s, e in self.pairs.get(name, [])]

    def count(self, name):
        return len(self.pairs.get(name, []))


def workload_name(wl) -> str:
    return f"{wl.name}: R={wl.R} E={wl.E} K={wl.K} S={wl.S} H={wl.H} B={wl.B}"


def time_layer(mp, wl, rt, hidden, buf, out, dev, iters, peak, graph=False):
    """One MoE layer's plan -> dispatch -> combine on routing ``rt``: CUDA-event
    times of each call (mean over ``iters`` eager layers, after 3 warm-up
    layers) and, with ``graph``, the whole layer replayed from a CUDA graph
    (mean over 50 replays).  Returns the point's line."""
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    p = mp.Plan(cfg, dev)
    # the plan block and its zero-filled workspace were made on the default
    # stream: finish that before a capture stream uses them
    torch.cuda.synchronize()
    for _ in range(3):
        mp.plan(cfg, rt.topk_idx, out=p)
        mp.dispatch(cfg, p, hidden, buf)
        mp.combine(cfg, p, buf, rt.weights, out)
    torch.cuda.synchronize()
    st = Timer()
    for _ in range(iters):
        e = st.mark("plan"); mp.plan(cfg, rt.topk_idx, out=p); e.record()
        e = st.mark("dispatch"); mp.dispatch(cfg, p, hidden, buf); e.record()
        e = st.mark("combine"); mp.combine(cfg, p, buf, rt.weights, out); e.record()
    torch.cuda.synchronize()
    pd, pc, pp = (st.total_ms(n) / iters for n in ("dispatch", "combine", "plan"))
    inf = p.info()
    gd = bytes_dispatch(wl) / (pd * 1e-3) / 1e9
    gc = bytes_combine(wl) / (pc * 1e-3) / 1e9
    pt = {"maxvio": round(rt.maxvio, 3), "planner_us": round(pp * 1e3, 2),
          "dispatch_us": round(pd * 1e3, 2), "combine_us": round(pc * 1e3, 2),
          "dispatch_GB/s": round(gd, 1), "combine_GB/s": round(gc, 1),
          "dispatch_frac": round(gd / peak, 4), "combine_frac": round(gc / peak, 4),
          "dispatch+combine_tok/s": round(wl.tokens / ((pd + pc) * 1e-3)),
          "n_rep": inf["n_rep"], "n_overflow": inf["n_overflow"],
          "max_rep_per_rank": inf["max_rep_per_rank"],
          # plan quality: any exact plan needs at least max(pieces, receivers)
          # replicas; the greedy makes at most pieces + receivers - 1
          "n_rep_bounds": [max(inf["n_pieces"], inf["n_receivers"]),
                           max(inf["n_pieces"] + inf["n_receivers"] - 1, 0)],
          "remote_pair_frac": round(inf["n_remote_pairs"] / wl.pairs, 4),
          "hottest_expert_pairs": W.hottest_expert_count(rt.maxvio, wl.S, wl.K, wl.R, wl.E)}
    if graph:
        gs_ = torch.cuda.Stream()
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gs_, capture_error_mode="thread_local"):
                mp.plan(cfg, rt.topk_idx, out=p)
                mp.dispatch(cfg, p, hidden, buf)
                mp.combine(cfg, p, buf, rt.weights, out)
            for _ in range(5):
                g.replay()
            torch.cuda.synchronize()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record()
            for _ in range(50):
                g.replay()
            g1.record()
            torch.cuda.synchronize()
            us = g0.elapsed_time(g1) / 50 * 1e3
            pt["graph_layer_us"] = round(us, 2)
            pt["dispatch+combine_GB/s_in_graph"] = round(
                (bytes_dispatch(wl) + bytes_combine(wl)) / (us * 1e-6) / 1e9, 1)
            del g
        except RuntimeError as exc:  # report the eager numbers if capture is refused
            pt["graph_error"] = str(exc)[:200]
            torch.cuda.synchronize()
    del p
    return pt


def run_ours(args, world, rank, local):
    from load_balancing_moonep_b200 import moonep as mp

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS[args.workload]
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    peak, peak_kind = measured_peaks()

    r = W.routing(wl, args.maxvio, seed=rank, device=dev)
    hidden = W.hidden_states(wl, seed=1 + rank, device=dev)
    dy = W.bf16_normal((wl.tokens, wl.H), seed=3 + rank, device=dev)
    buf = torch.empty((wl.R, wl.C, wl.H), dtype=torch.bfloat16, device=dev)
    dy_buf = torch.empty_like(buf)
    out = torch.empty((wl.tokens, wl.H), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((wl.tokens, wl.K), dtype=torch.float32, device=dev)
    plan = mp.Plan(cfg, dev)

    # replica gradients: the full gate+up+down size if it fits, else one projection
    P = wl.grad_elems if wl.H_ffn else 0
    reduce_note = "gate+up+down per expert"
    if P:
        free, _ = torch.cuda.mem_get_info(dev)
        need = 4 * P * (wl.R * wl.B + wl.E)
        if need > free - (6 << 30):
            P = wl.H * wl.H_ffn
            reduce_note = "one projection per expert (device memory)"
        rb = W.f32_normal((wl.R, wl.B, P), seed=4 + rank, device=dev, std=1e-3)
        hg = W.f32_normal((wl.E, P), seed=5 + rank, device=dev, std=1e-3)

    def step(tm: Timer | None):
        ev = tm.mark("plan") if tm else None
        mp.plan(cfg, r.topk_idx, out=plan)
        if tm:
            ev.record()
            ev = tm.mark("dispatch")
        mp.dispatch(cfg, plan, hidden, buf)
        if tm:
            ev.record()
            ev = tm.mark("combine")
        mp.combine(cfg, plan, buf, r.weights, out)
        if tm:
            ev.record()
            ev = tm.mark("combine_bwd")
        mp.combine_backward(cfg, plan, dy, r.weights, buf, dy_buf, dw)
        if tm:
            ev.record()
        if P:
            if tm:
                ev = tm.mark("reduce")
            mp.reduce_replica_grads(cfg, plan, rb, hg)
            if tm:
                ev.record()

    # the clock sampler starts before the warm-up: its start-up once delayed
    # the first timed plan call by about 45 us
    sampler = ClockSampler(smi_index(local))
    sampler.start()
    sampler.wait_first()
    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()
    info = plan.info()
    barrier(world)
    torch.cuda.synchronize()
    tm = Timer()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        step(tm)
    t_end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    step_ms_local = t_start.elapsed_time(t_end) / args.steps
    ms_per_step = max_over_ranks(world, step_ms_local)

    # this library's kernels in one untimed step
    launches_per_step, launches_how = count_library_launches(lambda: step(None))
    if launches_per_step is None:  # no profiler: the planner's one kernel and the data kernels
        launches_per_step = 1 + 1 + 1 + 1 + (1 if P else 0)
        launches_how = "static count (" + launches_how + ")"

    # the same step with the other planner, for comparison (its plan time
    # only; the data kernels do not depend on which planner made the plan)
    other = 1 - mp.set_plan_path(1 - args.plan_path)
    for _ in range(args.warmup):
        step(None)
    tm2 = Timer()
    for _ in range(args.steps):
        step(tm2)
    torch.cuda.synchronize()
    mp.set_plan_path(args.plan_path)
    other_plan_us = max_over_ranks(world, statistics.median(tm2.times_ms("plan"))) * 1e3
    plan_steps_us = [round(x * 1e3, 2) for x in tm.times_ms("plan")]
    plan_median_us = max_over_ranks(world, statistics.median(tm.times_ms("plan"))) * 1e3

    k = args.steps
    t = {n: tm.total_ms(n) / k for n in ("plan", "dispatch", "combine", "combine_bwd", "reduce")
         if tm.count(n)}
    dc_ms = max_over_ranks(world, t["dispatch"] + t["combine"])
    dc_bytes = (bytes_dispatch(wl) + bytes_combine(wl)) * world
    value = dc_bytes / (dc_ms * 1e-3) / 1e9

    n_pref = info["n_rep"] - info["n_overflow"]
    kb = {"plan": bytes_plan(wl), "dispatch": bytes_dispatch(wl), "combine": bytes_combine(wl),
          "combine_bwd": bytes_combine_bwd(wl)}
    if P:
        kb["reduce"] = bytes_reduce(n_pref, info["n_rep_experts"], P)
    ratio = ncu_traffic_ratio()
    traffic = {n: int(round(ratio[n] * b)) for n, b in kb.items() if n in ratio}
    kernels = {}
    for n, ms in t.items():
        gbs = kb[n] / (ms * 1e-3) / 1e9
        kernels[n] = {"ms": round(ms, 4), "bytes": kb[n], "GB/s": round(gbs, 1),
                      "frac": round(gbs / peak, 4), "traffic": traffic.get(n)}
    kernels["plan"]["us"] = round(t["plan"] * 1e3, 2)
    dom = max((n for n in t if n != "plan"), key=lambda n: t[n])
    roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["GB/s"], "peak": peak,
                "peak_kind": peak_kind + " (MEASURED_PEAKS.json hbm_gbs, copy read+write)",
                "unit": "GB/s", "frac": kernels[dom]["frac"], "traffic": traffic.get(dom),
                "traffic_how": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the "
                                "reduced-size profile case (profiles/ncu_traffic.json), scaled to this "
                                "launch by algorithmic bytes")}

    # maxvio sweep of the large shape (the Zipf sweep, then the adversarial
    # placement with all hot experts on rank 0)
    sweep = []
    if not args.no_sweep:
        for mv, adv in [(m, False) for m in wl.sweep] + [(max(wl.sweep), True)]:
            rs = W.routing(wl, mv, seed=rank, device=dev, adversarial=adv)
            pt = time_layer(mp, wl, rs, hidden, buf, out, dev, args.sweep_iters, peak)
            pt["adversarial"] = adv
            sweep.append(pt)

    # end to end through the public API with pinned host buffers: every step
    # copies its routing, weights and hidden states in and its output out.
    # Double-buffered and pipelined on three streams, so step i+1's inputs
    # and step i-1's output cross PCIe while step i runs.
    e2e = None
    if not args.no_e2e:
        nb = 2
        h_topk = [r.topk_idx.cpu().pin_memory() for _ in range(nb)]
        h_w = [r.weights.cpu().pin_memory() for _ in range(nb)]
        h_hidden = [hidden.cpu().pin_memory() for _ in range(nb)]
        h_out = [torch.empty((wl.tokens, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
        d_topk = [torch.empty_like(r.topk_idx) for _ in range(nb)]
        d_w = [torch.empty_like(r.weights) for _ in range(nb)]
        d_hidden = [hidden] + [torch.empty_like(hidden) for _ in range(nb - 1)]
        d_out = [out] + [torch.empty_like(out) for _ in range(nb - 1)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_used = [torch.cuda.Event() for _ in range(nb)]   # inputs consumed
        ev_done = [torch.cuda.Event() for _ in range(nb)]   # output written
        ev_read = [torch.cuda.Event() for _ in range(nb)]   # output copied out
        torch.cuda.synchronize()  # inputs, plan and buffers ready before the side streams start
        for b in range(nb):
            for ev in (ev_used[b], ev_read[b]):
                ev.record(s_cmp)

        def e2e_step(i):
            b = i % nb
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_used[b])
                d_topk[b].copy_(h_topk[b], non_blocking=True)
                d_w[b].copy_(h_w[b], non_blocking=True)
                d_hidden[b].copy_(h_hidden[b], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                s_cmp.wait_event(ev_read[b])
                mp.plan(cfg, d_topk[b], out=plan, stream=s_cmp)
                mp.dispatch(cfg, plan, d_hidden[b], buf, stream=s_cmp)
                mp.combine(cfg, plan, buf, d_w[b], d_out[b], stream=s_cmp)
                ev_used[b].record(s_cmp)
                ev_done[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                h_out[b].copy_(d_out[b], non_blocking=True)
                ev_read[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(4, min(args.steps, 10))
        a.record(s_in)
        s_cmp.wait_event(a)
        s_out.wait_event(a)
        for i in range(n_e2e):
            e2e_step(i)
        b_.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(world, a.elapsed_time(b_) / n_e2e)
        e2e = {"value": round(dc_bytes / (e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
               "ms_per_step": round(e_ms, 3),
               "h2d_bytes_per_step": int(h_topk[0].numel() * 4 + h_w[0].numel() * 4 + h_hidden[0].numel() * 2),
               "d2h_bytes_per_step": int(h_out[0].numel() * 2),
               "what": ("pinned host topk/weights/hidden -> plan -> dispatch -> combine -> pinned host "
                        "out, every step; double-buffered, copies of neighbouring steps overlap")}
        del d_topk, d_w, d_hidden, d_out

    # the other workloads, each across its maxvio sweep: the mid shape, the
    # pages' own sweep shape (EP=8, maxvio 0.2, 1, 10, 20), the tiny shape
    # (latency, L2-resident) and the decode shape (latency, each layer also
    # replayed from a CUDA graph)
    workloads = {}
    if not args.no_sweep:
        for wname, graph in (("mid", False), ("ep8", False), ("tiny", True)):
            owl = W.WORKLOADS[wname]
            oh = W.hidden_states(owl, seed=12 + rank, device=dev)
            obuf = torch.empty((owl.R, owl.C, owl.H), dtype=torch.bfloat16, device=dev)
            oout = torch.empty((owl.tokens, owl.H), dtype=torch.bfloat16, device=dev)
            pts = []
            for mv in owl.sweep:
                orr = W.routing(owl, mv, seed=rank, device=dev)
                pts.append(time_layer(mp, owl, orr, oh, obuf, oout, dev, args.sweep_iters, peak, graph=graph))
            workloads[wname] = {"workload": workload_name(owl), "points": pts,
                                "l2": ("inputs within L2: latency" if owl.tokens * owl.H * 2 * (owl.K + 1) < L2_BYTES
                                       else "buffers larger than L2")}
            del oh, obuf, oout

    # over-budget routing (one empty rank, the rest evenly overloaded): the
    # planner without and with the relay cascade, and the data kernels over
    # the cascade's plan
    cascade = None
    if not args.no_sweep:
        cr = W.over_budget_routing(wl, seed=rank, device=dev)
        cascade = {"workload": f"{wl.name} shape, rank 0's experts empty, the other "
                               f"{wl.R - 1} ranks evenly overloaded", "points": []}
        for flags in (0, mp.FLAG_CASCADE):
            ccfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=flags)
            cp = mp.Plan(ccfg, dev)
            for _ in range(3):
                mp.plan(ccfg, cr.topk_idx, out=cp)
                mp.dispatch(ccfg, cp, hidden, buf)
                mp.combine(ccfg, cp, buf, cr.weights, out)
            torch.cuda.synchronize()
            st = Timer()
            for _ in range(args.sweep_iters):
                e = st.mark("plan"); mp.plan(ccfg, cr.topk_idx, out=cp); e.record()
                e = st.mark("dispatch"); mp.dispatch(ccfg, cp, hidden, buf); e.record()
                e = st.mark("combine"); mp.combine(ccfg, cp, buf, cr.weights, out); e.record()
            torch.cuda.synchronize()
            it = args.sweep_iters
            pd, pc, pp = st.total_ms("dispatch") / it, st.total_ms("combine") / it, st.total_ms("plan") / it
            inf = cp.info()
            cascade["points"].append({
                "cascade": bool(flags), "planner_us": round(pp * 1e3, 2),
                "dispatch_GB/s": round(bytes_dispatch(wl) / (pd * 1e-3) / 1e9, 1),
                "combine_GB/s": round(bytes_combine(wl) / (pc * 1e-3) / 1e9, 1),
                "status": inf["status"], "n_rep": inf["n_rep"], "n_overflow": inf["n_overflow"],
                "max_rep_per_rank": inf["max_rep_per_rank"],
                "remote_pair_frac": round(inf["n_remote_pairs"] / wl.pairs, 4)})
            del cp
        del cr

    # decode shape (latency-bound): plan + dispatch + combine of one MoE layer
    # replayed from a CUDA graph, next to the eager per-kernel times, at each
    # point of its sweep
    decode = None
    if not args.no_decode:
        dwl = W.WORKLOADS["decode"]
        dh = W.hidden_states(dwl, seed=11 + rank, device=dev)
        dbuf = torch.empty((dwl.R, dwl.C, dwl.H), dtype=torch.bfloat16, device=dev)
        dout = torch.empty((dwl.tokens, dwl.H), dtype=torch.bfloat16, device=dev)
        pts = []
        for mv in dwl.sweep:
            dr = W.routing(dwl, mv, seed=rank, device=dev)
            pts.append(time_layer(mp, dwl, dr, dh, dbuf, dout, dev, 20, peak, graph=True))
        decode = {"workload": workload_name(dwl) + ", one hot expert", "points": pts,
                  "l2": "buffers larger than L2 (940 MB)"}
        del dbuf, dout, dh

    # replica weight prefetch (a next-row step, timed on its own after the
    # step: its 68 GB of weights and pool fit once the reduce buffers are freed)
    if P and not args.no_prefetch:
        del rb, hg
        torch.cuda.empty_cache()
        Pw = wl.grad_elems
        weights = W.bf16_normal((wl.E, Pw), seed=7 + rank, device=dev)
        pool = torch.empty((wl.R, wl.B, Pw), dtype=torch.bfloat16, device=dev)
        wrow = torch.empty((wl.R, wl.E), dtype=torch.int32, device=dev)
        for _ in range(2):
            mp.prefetch_replicas(cfg, plan, weights, pool, wrow)
        torch.cuda.synchronize()
        pt = Timer()
        for _ in range(5):
            ev = pt.mark("prefetch")
            mp.prefetch_replicas(cfg, plan, weights, pool, wrow)
            ev.record()
        torch.cuda.synchronize()
        pms = pt.total_ms("prefetch") / 5
        pbytes = bytes_prefetch(n_pref, info["n_rep_experts"], Pw, wl)
        ptraffic = int(round(ratio["prefetch"] * pbytes)) if "prefetch" in ratio else None
        kernels["prefetch"] = {"ms": round(pms, 4), "bytes": pbytes, "GB/s": round(pbytes / (pms * 1e-3) / 1e9, 1),
                               "frac": round(pbytes / (pms * 1e-3) / 1e9 / peak, 4), "traffic": ptraffic,
                               "in_step": False,
                               "what": (f"{n_pref} replicas of {info['n_rep_experts']} experts x {Pw} bf16 "
                                        "(gate+up+down) copied into the pool, each source row read once")}
        del weights, pool, wrow
        torch.cuda.empty_cache()

    # expert parallelism's calls on one GPU: every rank's count and plan from
    # the stacked counts rows (what the all-gather leaves), then its dispatch
    # and combine through an array of R per-rank row-buffer pointers (here
    # the R slices of the one buffer), one launch per rank as one process
    # per GPU would issue them
    ep = None
    if not args.no_ep:
        eplans = [mp.Plan(cfg, dev, ep=True) for _ in range(wl.R)]
        counts_all = torch.empty((wl.R, wl.E + 1), dtype=torch.int32, device=dev)
        tl = [r.topk_idx[k * wl.S:(k + 1) * wl.S].contiguous() for k in range(wl.R)]
        hl = [hidden[k * wl.S:(k + 1) * wl.S] for k in range(wl.R)]
        wloc = [r.weights[k * wl.S:(k + 1) * wl.S].contiguous() for k in range(wl.R)]
        ol = [out[k * wl.S:(k + 1) * wl.S] for k in range(wl.R)]
        bptr = mp.pointer_array([buf[k] for k in range(wl.R)])
        torch.cuda.synchronize()

        def ep_layer(tm):
            for k in range(wl.R):
                e = tm.mark("count") if tm and k == 0 else None
                mp.ep_count(cfg, tl[k], eplans[k], counts_row=counts_all[k])
                if e:
                    e.record()
            for k in range(wl.R):
                if tm and k == 0:
                    # keep the GPU busy while the host enqueues the plan, so
                    # the events time the device, not the host's launch path
                    torch.cuda._sleep(SPACER_CYCLES)
                e = tm.mark("plan") if tm and k == 0 else None
                mp.ep_plan(cfg, k, tl[k], counts_all, eplans[k])
                if e:
                    e.record()
            e = tm.mark("dispatch") if tm else None
            for k in range(wl.R):
                mp.ep_dispatch(cfg, eplans[k], hl[k], bptr)
            if e:
                e.record()
                e = tm.mark("combine")
            for k in range(wl.R):
                mp.ep_combine(cfg, eplans[k], bptr, wloc[k], ol[k])
            if e:
                e.record()

        for _ in range(3):
            ep_layer(None)
        torch.cuda.synchronize()
        et = Timer()
        for _ in range(args.sweep_iters):
            ep_layer(et)
        torch.cuda.synchronize()
        it = args.sweep_iters
        # rank 0's plan with the other expert-parallel planner, timed the same way
        other_ep = 1 - mp.set_plan_path(1 - args.plan_path)
        ot = Timer()
        for _ in range(args.sweep_iters):
            ep_layer(ot)
        torch.cuda.synchronize()
        mp.set_plan_path(args.plan_path)
        pd, pc = et.total_ms("dispatch") / it, et.total_ms("combine") / it
        einf = eplans[0].info()
        gd = bytes_dispatch(wl) / (pd * 1e-3) / 1e9
        gc = bytes_combine(wl) / (pc * 1e-3) / 1e9
        # locality-aware intervals: the pairs kept on their source rank, with
        # and without the flag, on the pages' EP = 8 shape at maxvio 20 and on
        # this shape at maxvio 3 (plans only)
        locality = []
        for lname, lmv in (("ep8", 20.0), (wl.name, 3.0)):
            lwl = W.WORKLOADS[lname]
            lr = W.routing(lwl, lmv, seed=rank, device=dev)
            row = {"workload": workload_name(lwl), "maxvio": round(lr.maxvio, 3)}
            for lflags, key in ((0, "remote_pair_frac"), (mp.FLAG_LOCALITY, "remote_pair_frac_locality")):
                lcfg = mp.Config(R=lwl.R, E=lwl.E, K=lwl.K, S=lwl.S, H=lwl.H, B=lwl.B, flags=lflags)
                lps = [mp.Plan(lcfg, dev, ep=True) for _ in range(lwl.R)]
                lca = torch.empty((lwl.R, lwl.E + 1), dtype=torch.int32, device=dev)
                ltl = [lr.topk_idx[k * lwl.S:(k + 1) * lwl.S].contiguous() for k in range(lwl.R)]
                torch.cuda.synchronize()
                for k in range(lwl.R):
                    mp.ep_count(lcfg, ltl[k], lps[k], counts_row=lca[k])
                lt = Timer()
                for rep_ in range(4):  # the first call warms up; the median of the other three
                    for k in range(lwl.R):
                        if k == 0:
                            torch.cuda._sleep(SPACER_CYCLES)
                        e = lt.mark("plan") if k == 0 else None
                        mp.ep_plan(lcfg, k, ltl[k], lca, lps[k])
                        if e:
                            e.record()
                torch.cuda.synchronize()
                row[key] = round(sum(q.info()["n_remote_pairs"] for q in lps) / lwl.pairs, 4)
                row["plan_us" + ("_locality" if lflags else "")] = round(
                    statistics.median(lt.times_ms("plan")[1:]) * 1e3, 2)
                del lps
            locality.append(row)
        ep = {"what": (f"{wl.R} ranks on one GPU: each rank's ep_count and ep_plan (rank 0 timed), then "
                       f"{wl.R} ep_dispatch and {wl.R} ep_combine launches through per-rank row pointers"),
              "count_us": round(et.total_ms("count") / it * 1e3, 2),
              "plan_us": round(statistics.median(et.times_ms("plan")) * 1e3, 2),
              "plan_us_other_path": {"path": "two-kernel" if other_ep == 1 else "one-kernel",
                                     "us": round(statistics.median(ot.times_ms("plan")) * 1e3, 2)},
              "plan_timing": "rank 0's plan after a device-side sleep that covers the host's launch path",
              "dispatch_GB/s": round(gd, 1), "combine_GB/s": round(gc, 1),
              "dispatch_frac": round(gd / peak, 4), "combine_frac": round(gc / peak, 4),
              "rank0_remote_pair_frac": round(einf["n_remote_pairs"] / (wl.S * wl.K), 4),
              "status": einf["status"], "locality": locality}
        del eplans, bptr

    # the CPU oracle on a bounded sample (rank 0, one GPU only): the
    # single-threaded oracle, then the same loops built with OpenMP on all of
    # the host's cores
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        topk_np = r.topk_idx.cpu().numpy()
        w_np = r.weights.cpu().numpy()
        tokens = sample_tokens(wl, args.ref_tokens)
        hid = W.bits(hidden[: len(tokens)])
        y = W.bits(W.bf16_normal((len(tokens) * wl.K, wl.H), seed=2, device="cpu"))
        ncores = host_cores()
        # repeat the bounded sample until about 10 s of CPU work
        reps, ds_tot, db_tot, ps_ = 0, 0.0, 0.0, 0.0
        while ds_tot < 10.0 and reps < 50:
            ps_, ds_, db_ = oracle_sample(wl, topk_np, w_np, hid, tokens, y)
            ds_tot += ds_
            db_tot += db_
            reps += 1
        rs_, rb_ = oracle_reduce_sample(wl, topk_np, 1 << 18)
        olib, nthr = oracle.openmp_lib(ncores)
        oreps, ods, odb = 0, 0.0, 0.0
        while ods < 5.0 and oreps < 200:
            _, d_, b_ = oracle_sample(wl, topk_np, w_np, hid, tokens, y, lib=olib, plan=False)
            ods += d_
            odb += b_
            oreps += 1
        ors_, orb_ = oracle_reduce_sample(wl, topk_np, 1 << 18, lib=olib)
        tok = len(tokens)
        gpu_tok = wl.tokens / ((t["dispatch"] + t["combine"]) * 1e-3)
        cpu = {"value": round(db_tot / ds_tot / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": (f"{reps} x dispatch+combine of the first {tok} of {wl.tokens} tokens "
                          f"({ds_tot:.1f} s); plan over all {wl.pairs} pairs took {ps_ * 1e3:.0f} ms; "
                          "single-threaded C"),
               "host_cores": ncores,
               "dispatch+combine_tok/s": round(reps * tok / ds_tot),
               "planner_us": round(ps_ * 1e6, 1),
               "reduce_GB/s": round(rb_ / rs_ / 1e9, 4),
               "openmp": {"value": round(odb / ods / 1e9, 4), "unit": UNIT, "threads": nthr,
                          "dispatch+combine_tok/s": round(oreps * tok / ods),
                          "reduce_GB/s": round(orb_ / ors_ / 1e9, 4),
                          "sample": (f"{oreps} x the same token sample ({ods:.1f} s), the oracle's loops "
                                     f"built with OpenMP over tokens on {nthr} threads; reduce over "
                                     f"elements, rows of 2^18 of the {wl.grad_elems} gradient elements")},
               "gpu_dispatch+combine_tok/s": round(gpu_tok)}

    cfgd = workload_config(wl, r, args)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfgd,
        "frac_of_peak": round(value / world / peak, 4),
        # the median over the timed steps (kernels.plan is their mean): a
        # single slow call, e.g. as the clock sampler starts, moves the mean
        "planner_us": round(plan_median_us, 2),
        "planner_us_steps": plan_steps_us,
        "planner_us_other_path": {"path": "two-kernel" if other == 1 else "one-kernel",
                                  "us": round(other_plan_us, 2)},
        "roofline": roofline, "kernels": kernels, "sweep": sweep,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_how": launches_how,
        "decode": decode, "workloads": workloads, "ep_one_gpu": ep,
        "cascade": cascade, "clocks": clocks, "plan_info": info,
        "reduce": (f"P={P} fp32 ({reduce_note}), {n_pref} prefetched replicas over "
                   f"{info['n_rep_experts']} experts"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# The ncu profile case of each kernel: (workload, tokens per rank S, elements
# per expert row P).  The data kernels run the large training shape with
# fewer tokens per rank; the reduce and the prefetch run the tiny shape with
# long rows, so that the few rows its plan touches still move several times
# the 126 MB L2 while every buffer of the case stays within a few GB.
PROFILE_CASES = {
    "dispatch": ("large", 512, 0), "combine": ("large", 512, 0), "combine_bwd": ("large", 512, 0),
    "reduce": ("tiny", 256, 1 << 25), "prefetch": ("tiny", 256, 1 << 26), "plan": ("large", 4096, 0),
}
PROFILE_KERNELS = tuple(PROFILE_CASES)


def run_profile_case(args):
    """--profile KERNEL: the kernel's reduced-size profile case
    (PROFILE_CASES; --profile-S / --profile-P override S and P) for ncu
    captures of ONE kernel: the plan, then two launches of that kernel (the
    capture skips the first: ``-k regex:moonep::<kernel> -s 1 -c 1``).  Only
    the buffers that kernel needs are allocated: at most about 4 GB on the
    device.  Prints the case and the kernel's algorithmic bytes per launch
    (the same byte model as the timed run), no timing."""
    from load_balancing_moonep_b200 import moonep as mp
    kern = args.profile
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wname, S_case, P_case = PROFILE_CASES[kern]
    wl = W.WORKLOADS[wname].with_(S=args.profile_S or S_case)
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    r = W.routing(wl, args.maxvio, seed=0, device=dev)
    plan = mp.Plan(cfg, dev)
    mp.plan(cfg, r.topk_idx, out=plan)
    torch.cuda.synchronize()
    info = plan.info()
    n_pref = info["n_rep"] - info["n_overflow"]
    P = args.profile_P or P_case
    if kern == "plan":
        for _ in range(2):
            mp.plan(cfg, r.topk_idx, out=plan)
        alg = bytes_plan(wl)
    elif kern == "dispatch":
        hidden = W.hidden_states(wl, seed=1, device=dev)
        buf = torch.empty((wl.R, wl.C, wl.H), dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            mp.dispatch(cfg, plan, hidden, buf)
        alg = bytes_dispatch(wl)
    elif kern == "combine":
        y = W.bf16_normal((wl.R, wl.C, wl.H), seed=2, device=dev)
        out = torch.empty((wl.tokens, wl.H), dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            mp.combine(cfg, plan, y, r.weights, out)
        alg = bytes_combine(wl)
    elif kern == "combine_bwd":
        y = W.bf16_normal((wl.R, wl.C, wl.H), seed=2, device=dev)
        dy = W.bf16_normal((wl.tokens, wl.H), seed=3, device=dev)
        dy_buf = torch.empty_like(y)
        for _ in range(2):
            mp.combine_backward(cfg, plan, dy, r.weights, y, dy_buf)
        alg = bytes_combine_bwd(wl)
    elif kern == "reduce":
        rb = W.f32_normal((wl.R, wl.B, P), seed=4, device=dev, std=1e-3)
        hg = W.f32_normal((wl.E, P), seed=5, device=dev, std=1e-3)
        for _ in range(2):
            mp.reduce_replica_grads(cfg, plan, rb, hg)
        alg = bytes_reduce(n_pref, info["n_rep_experts"], P)
    elif kern == "prefetch":
        weights = W.bf16_normal((wl.E, P), seed=7, device=dev)
        pool = torch.empty((wl.R, wl.B, P), dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            mp.prefetch_replicas(cfg, plan, weights, pool)
        alg = bytes_prefetch(n_pref, info["n_rep_experts"], P, wl)
    else:
        raise SystemExit(f"--profile: unknown kernel {kern}")
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": f"{wl.name} S={wl.S}" + (f" P={P}" if P else ""), "kernel": kern,
                      "tokens": wl.tokens, "P": P, "alg_bytes_per_launch": alg,
                      "n_rep": info["n_rep"], "n_overflow": info["n_overflow"],
                      "n_rep_experts": info["n_rep_experts"],
                      "device_GB": round(torch.cuda.max_memory_allocated() / 1e9, 2)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="large", choices=sorted(W.WORKLOADS))
    ap.add_argument("--maxvio", type=float, default=1.0)
    ap.add_argument("--sweep-iters", type=int, default=10)
    ap.add_argument("--ref-tokens", type=int, default=8192)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefetch", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-ep", action="store_true")
    ap.add_argument("--profile", default=None, choices=PROFILE_KERNELS,
                    help="run one kernel twice on a reduced-size case of a few GB (for ncu)")
    ap.add_argument("--profile-S", type=int, default=0, help="tokens per rank (0: the kernel's case)")
    ap.add_argument("--profile-P", type=int, default=0,
                    help="elements per expert row for reduce / prefetch (0: the kernel's case)")
    ap.add_argument("--plan-path", type=int, default=0, choices=(0, 1),
                    help="0: the one-kernel planner where it fits (the library's default); "
                         "1: the two-kernel planner (moonep_set_plan_path)")
    args = ap.parse_args()
    if args.impl != "reference" or args.profile:
        from load_balancing_moonep_b200 import moonep as mp
        mp.set_plan_path(args.plan_path)
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3:
        log("warmup raised to 3 (timing rule)")
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
