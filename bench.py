#!/usr/bin/env python3
"""Benchmark of the MoE layout -> dispatch -> combine hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline] [--no-e2e] [--no-decode]
                    [--no-backward] [--no-overlap] [--no-ranks] [--ep]

A step is one pass of the whole path over one batch: ep_layout (2 kernels),
ep_dispatch (FP8 e4m3 or BF16), ep_combine (BF16), all through the C ABI.
The default workload is the one the metric is quoted on: 8192 tokens,
hidden 7168, top-8 of 256 experts with group-limited gating (8 groups, top-4
groups, Zipf(1.0) bias), 64 virtual ranks, FP8 dispatch, BF16 combine.

Timing: inputs resident in HBM; L2 flushed (256 MiB write) before every
timed step; CUDA events on the launching stream around each call; W warm-up
steps; K timed steps bracketed by barrier + synchronize; max over ranks.
value = algorithmic bytes of all ranks' steps / time (GB/s).  Multi-GPU runs
are independent replicas (each rank its own batch, seed + rank): the path
has no exchange step on one node's virtual ranks, so there is no collective.

`--ep` adds expert parallelism across the job's GPUs (peer dispatch and
combine between the ranks, NCCL collectives between the phases) as an extra
object of the same line.

`--impl reference` times the CPU oracle (the plain single-threaded C
implementation under oracle/) on a bounded sample of the same workload per
step, shrunk until the whole run fits a fixed time budget.
"""
from __future__ import annotations

import argparse
import datetime
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
sys.path.insert(0, ROOT)

from combine_ep_layout_10_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
GPU_LEAD_CYCLES = 1_000_000  # ~0.5 ms spin before each timed step
CALL_KERNELS = 2             # dispatch and combine launch one kernel each;
                             # the layout's count comes back on its handle
HBM_FALLBACK_GBS = 6650.0
# The reference arm's projected run time (its per-step sample shrinks to fit).
REFERENCE_BUDGET_S = float(os.environ.get("EP_BENCH_REFERENCE_BUDGET_S", "150"))

# DRAM traffic per launch from one ncu capture, keyed by the sha256 of the
# kernel source it was taken on (stale -> reported as null).
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch each on the
    # metric workload (one ncu capture per kernel, keyed to the kernel source)
    ("group_limited", "combine"): {"sha": "61964820f31d742f", "bytes": 940124416 + 72721408},
    ("group_limited", "dispatch"): {"sha": "70e5e8aacbf867c8", "bytes": 117771776 + 425458432},
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=W.METRIC_WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-backward", action="store_true")
    p.add_argument("--no-overlap", action="store_true")
    p.add_argument("--no-gemm-layout", action="store_true")
    p.add_argument("--no-ranks", action="store_true")
    p.add_argument("--ep", action="store_true",
                   help="also run expert parallelism across the job's GPUs (peer stores/loads)")
    p.add_argument("--seed", type=int, default=0)
    return p.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes (exact reads + writes each kernel must do)
# ---------------------------------------------------------------------------

def algorithmic_bytes(w: W.Workload, V: int, n_rows: int) -> dict:
    T, H, k, E, R = w.T, w.H, w.k, w.E, w.R
    layout = T * k * 4 + E * 4 + R * 4 + T * R + T * k * 4 + n_rows * 4 + (E + 1) * 4 + (R + 1) * 4
    if w.fp8:
        dispatch = T * H * 2 + T * k * 4 + V * H + V * (H // 128) * 4
    else:
        dispatch = T * H * 2 + T * k * 4 + V * H * 2
    combine = V * H * 2 + T * k * 4 + T * k * 4 + T * H * 2
    return {"layout": layout, "dispatch": dispatch, "combine": combine,
            "step": layout + dispatch + combine}


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": HBM_FALLBACK_GBS, "source": "fallback"}


def source_sha(name: str) -> str:
    p = os.path.join(ROOT, "combine_ep_layout_10_b200", "csrc", name)
    with open(p, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons sampled every 10 ms by NVML (reads
    only) on the benchmark's GPU; nvidia-smi at 100 ms if NVML is missing."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []          # (wall time, sm MHz, max sm MHz, reasons bitmask)
        self._stop = threading.Event()
        self.thread = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.source = "nvml"

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                             smax, int(reasons_fn(h))))
                    except Exception:
                        pass
                    time.sleep(0.01)
        except Exception:
            self.source = "nvidia-smi"
            fields = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
                      "clocks_event_reasons.hw_thermal_slowdown",
                      "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

            def run():
                try:
                    proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev),
                                             "--query-gpu=" + ",".join(fields),
                                             "--format=csv,noheader,nounits", "-lms", "100"],
                                            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                except Exception:
                    return
                bits = [0x8, 0x40, 0x20, 0x4]
                for line in proc.stdout:
                    parts = [q.strip() for q in line.split(",")]
                    try:
                        mask = sum(b for b, v in zip(bits, parts[2:]) if v.lower().startswith("active"))
                        self.samples.append((time.time(), float(parts[0]), float(parts[1]), mask))
                    except (ValueError, IndexError):
                        pass
                    if self._stop.is_set():
                        break
                proc.terminate()
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self, window=None) -> dict:
        """Summarise the samples taken inside `window` (wall-clock start, end)."""
        self._stop.set()
        if self.thread:
            self.thread.join(timeout=5)
        sel = [x for x in self.samples if window is None or window[0] <= x[0] <= window[1]]
        reasons = sorted(n for n, b in self.REASONS.items() if any(x[3] & b for x in sel))
        return {"sm_mhz": statistics.median(x[1] for x in sel) if sel else None,
                "sm_max_mhz": max(x[2] for x in sel) if sel else None,
                "reasons": reasons, "samples": len(sel), "source": self.source}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------

class _StdoutToStderr:
    """Sends file descriptor 1 to stderr for a while: NCCL prints its version
    line on stdout when a communicator is created, and stdout must carry
    only the JSON result line."""

    def __enter__(self):
        sys.stdout.flush()
        self.saved = os.dup(1)
        os.dup2(2, 1)
        return self

    def __exit__(self, *exc):
        sys.stdout.flush()
        os.dup2(self.saved, 1)
        os.close(self.saved)
        return False


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (n_gpus, world))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        with _StdoutToStderr():
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(v: float, world: int, op: str) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def reduce_max(v: float, world: int) -> float:
    """Max over ranks (device times: the slowest replica sets the job time)."""
    return _reduce(v, world, "max")


def reduce_sum(v: float, world: int) -> float:
    """Sum over ranks (bytes: every replica's work counts)."""
    return _reduce(v, world, "sum")


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch."""
    return base + rank


def job_throughput(step_ms_local: float, bytes_per_step_local: float, steps: int, world: int):
    """Whole-job GB/s: all ranks' algorithmic bytes over the slowest rank's time."""
    step_ms = reduce_max(step_ms_local, world)
    total = reduce_sum(bytes_per_step_local * steps, world)
    return total / (step_ms * steps / 1e3) / 1e9, step_ms


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_sample_step(orc, w: W.Workload, x, idx, tw, n_tok: int, y_sample):
    """One oracle pass: full layout + dispatch/combine of the first n_tok tokens."""
    _, L = orc.layout(idx, w.E, w.R, w.align, w.capacity)
    pos = np.arange(n_tok * w.k, dtype=np.int32).reshape(n_tok, w.k)
    if w.fp8:
        orc.dispatch_fp8(x[:n_tok], pos, n_tok * w.k)
    else:
        orc.dispatch_bf16(x[:n_tok], pos, n_tok * w.k)
    orc.combine(y_sample, tw[:n_tok], pos)
    return L


def oracle_sample_inputs(w, seed, n_tok):
    x, idx, tw = W.make_routing(w, seed)
    y = W.make_expert_out(n_tok * w.k, w.H, seed + 1)
    return x, idx.numpy(), tw.numpy(), y


def oracle_bytes(w, n_tok, n_rows_full):
    sub = w.scaled(T=n_tok)
    b = algorithmic_bytes(sub, n_tok * w.k, n_tok * w.k)
    full_layout = algorithmic_bytes(w, w.T * w.k, n_rows_full)["layout"]
    return full_layout + b["dispatch"] + b["combine"]


def cpu_baseline(w: W.Workload, seed: int, budget_s: float = 12.0, n_tok: int = 2048) -> dict:
    import oracle as orc
    n_tok = min(n_tok, w.T)
    x, idx, tw, y = oracle_sample_inputs(w, seed, n_tok)
    n_rows = orc.max_recv_rows(w.T, w.k, w.E, w.align, w.capacity)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_sample_step(orc, w, x, idx, tw, n_tok, y)
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 50:
            break
    dt = time.perf_counter() - t0
    byts = oracle_bytes(w, n_tok, n_rows) * reps
    return {"value": byts / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d x (layout of all %d tokens + %s dispatch and BF16 combine of the first "
                      "%d tokens), %.1f s single-threaded C" % (reps, w.T, "FP8" if w.fp8 else "BF16",
                                                                 n_tok, dt),
            "host_cpu": host_cpu(),
            "all_cores": cpu_baseline_all_cores(w, x, idx, tw, y, n_tok, n_rows, budget_s / 2)}


def cpu_baseline_all_cores(w: W.Workload, x, idx, tw, y, n_tok: int, n_rows: int, budget_s: float) -> dict:
    """The same oracle, unchanged, over all host cores: the sample's tokens
    split into one contiguous shard per core, each shard's dispatch and
    combine run by its own thread (the C calls release the interpreter lock),
    the layout (a sequential definition) on one.  A reported baseline beside
    the single-core figure, not the target."""
    import oracle as orc
    from concurrent.futures import ThreadPoolExecutor
    cores = max(1, min(os.cpu_count() or 1, n_tok))
    bounds = [(i * n_tok // cores, (i + 1) * n_tok // cores) for i in range(cores)]
    bounds = [(a, b) for a, b in bounds if b > a]
    xs = [x[a:b].contiguous() for a, b in bounds]
    ts = [np.ascontiguousarray(tw[a:b]) for a, b in bounds]
    ys = [y[a * w.k:b * w.k].contiguous() for a, b in bounds]
    pos = [np.arange((b - a) * w.k, dtype=np.int32).reshape(b - a, w.k) for a, b in bounds]

    def shard(i):
        n = (bounds[i][1] - bounds[i][0]) * w.k
        if w.fp8:
            orc.dispatch_fp8(xs[i], pos[i], n)
        else:
            orc.dispatch_bf16(xs[i], pos[i], n)
        orc.combine(ys[i], ts[i], pos[i])

    with ThreadPoolExecutor(max_workers=len(bounds)) as pool:
        t0 = time.perf_counter()
        reps = 0
        while True:
            orc.layout(idx, w.E, w.R, w.align, w.capacity)
            list(pool.map(shard, range(len(bounds))))
            reps += 1
            if time.perf_counter() - t0 > budget_s or reps >= 100:
                break
        dt = time.perf_counter() - t0
    byts = oracle_bytes(w, n_tok, n_rows) * reps
    return {"value": byts / dt / 1e9, "unit": "GB/s", "cores": len(bounds), "kind": "oracle, token-sharded",
            "sample": "%d x (layout of all %d tokens on one thread + dispatch and combine of the first %d "
                      "tokens in %d shards, one thread each), %.1f s" % (reps, w.T, n_tok, len(bounds), dt)}


def host_cpu() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return "%s x%d" % (ln.split(":", 1)[1].strip(), os.cpu_count() or 0)
    except Exception:
        pass
    return "unknown"


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle as orc
    # Each step is a bounded sample: the dispatch and combine of the first
    # n_tok tokens, halved (down to 64) until the whole run's projected time
    # fits REFERENCE_BUDGET_S; the probes count as warm-up.
    n_tok = min(1024, w.T)
    x, idx, tw, y = oracle_sample_inputs(w, args.seed, n_tok)
    probes = 0
    while True:
        t0 = time.perf_counter()
        oracle_sample_step(orc, w, x, idx, tw, n_tok, y)
        probes += 1
        per_step = time.perf_counter() - t0
        if n_tok <= 64 or per_step * (args.steps + args.warmup) <= REFERENCE_BUDGET_S:
            break
        n_tok = max(64, n_tok // 2)
        x, idx, tw, y = oracle_sample_inputs(w, args.seed, n_tok)
    n_rows = orc.max_recv_rows(w.T, w.k, w.E, w.align, w.capacity)
    for _ in range(max(args.warmup - probes, 0)):
        oracle_sample_step(orc, w, x, idx, tw, n_tok, y)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(orc, w, x, idx, tw, n_tok, y)
    dt = time.perf_counter() - t0
    byts = oracle_bytes(w, n_tok, n_rows) * args.steps
    value = byts / dt / 1e9
    sample = ("each step: layout of all %d tokens + %s dispatch and BF16 combine of the first %d "
              "tokens (single-threaded C oracle)" % (w.T, "FP8" if w.fp8 else "BF16", n_tok))
    line = {
        "impl": "reference", "metric": "dispatch/combine HBM GB/s & % of peak; us/call at 8192 tok, "
                                       "H=7168, top-8", "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": storage_dtype(w), "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cpu": host_cpu()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def storage_dtype(w: W.Workload) -> str:
    """The bench line's dtype: fp32 arithmetic (the FP8 scale and 448/amax,
    the combine's fma chain), and the formats the data is stored in."""
    disp = "e4m3 + f32 scales" if w.fp8 else "bf16"
    return "f32 arithmetic; bf16 x -> %s dispatched; bf16 y -> bf16 combined" % disp


def workload_config(w: W.Workload, world: int) -> dict:
    return {"workload": w.name, "tokens": w.T, "hidden": w.H, "topk": w.k, "experts": w.E,
            "virtual_ranks": w.R, "dispatch": "fp8_e4m3 (fp32 scale / 128 ch)" if w.fp8 else "bf16",
            "combine": "bf16 (fp32 fma chain)", "capacity": w.capacity, "expert_alignment": w.align,
            "routing": w.routing,
            "l2": "flushed before every timed step (256 MiB write, then 256 MiB read to drain dirty lines)",
            "replicas": world, "parallelism": "replicas (no collective)"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def run_ours(args, w):
    from combine_ep_layout_10_b200 import build as B
    from combine_ep_layout_10_b200 import ep

    world, rank, local = dist_setup(args.gpus)
    if not os.path.exists(ep.LIB_PATH):
        B.build()
    ep.lib()
    dev = torch.device("cuda", local)
    seed = replica_seed(args.seed, rank)
    x_cpu, idx_cpu, tw_cpu = W.make_routing(w, seed)
    T, H, k, E, R = w.T, w.H, w.k, w.E, w.R
    n_rows = ep.ep_max_recv_rows(T, k, E, w.align, w.capacity)
    V = int((idx_cpu >= 0).sum())
    nbytes = algorithmic_bytes(w, V, n_rows)

    x = x_cpu.to(dev)
    idx = idx_cpu.to(dev)
    tw = tw_cpu.to(dev)
    g = torch.Generator(device=dev).manual_seed(seed + 1)
    y = torch.randn(n_rows, H, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    rdt = torch.float8_e4m3fn if w.fp8 else torch.bfloat16
    recv = torch.empty(n_rows, H, dtype=rdt, device=dev)
    scales = torch.empty(n_rows, H // 128, dtype=torch.float32, device=dev) if w.fp8 else None
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    cnt = torch.empty(E, dtype=torch.int32, device=dev)
    rtok = torch.empty(R, dtype=torch.int32, device=dev)
    in_rank = torch.empty(T, R, dtype=torch.uint8, device=dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # Write a buffer larger than L2, then read another one: the read
        # evicts the dirty lines (written back here, outside the timed window)
        # and leaves L2 holding clean, unrelated data.
        flush_w.zero_()
        flush_r.sum(dtype=torch.int64)

    def step(ev=None):
        """One layout -> dispatch -> combine.  ev: None, 2 events (step
        boundaries) or 4 events (one window per call)."""
        if ev is not None:
            # Let the host run ahead: the step's launches are all queued before
            # the GPU reaches ev[0], so the windows hold GPU time only (the
            # host issue time is reported separately as host_us_per_step).
            torch.cuda._sleep(GPU_LEAD_CYCLES)
            ev[0].record(stream)
        res = ep.ep_layout(idx, E, R, w.align, w.capacity, num_tokens_per_expert=cnt,
                           num_tokens_per_rank=rtok, is_token_in_rank=in_rank)
        if ev is not None and len(ev) == 4:
            ev[1].record(stream)
        ep.ep_dispatch(res.handle, x, w.fp8, recv, scales)
        if ev is not None and len(ev) == 4:
            ev[2].record(stream)
        ep.ep_combine(res.handle, y, tw, out)
        if ev is not None:
            ev[-1].record(stream)
        return res.handle

    for _ in range(max(args.warmup, 0)):
        flush_l2()
        step().free()
    torch.cuda.synchronize()
    assert step().check() == ep.EP_OK

    # Timed region: events at step boundaries only, so that nothing sits between
    # the step's kernels in the stream (the kernels use programmatic dependent
    # launch and may overlap their launch with the previous kernel's tail).
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.1)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    t0_wall = time.time()
    last = None
    launches = 0
    for i in range(args.steps):
        flush_l2()
        h = step(events[i])
        launches += h.layout_kernels + CALL_KERNELS
        if last is not None:
            last.free()
        last = h
    layout_kernels = last.layout_kernels
    torch.cuda.synchronize()
    barrier(world)
    wall1 = time.perf_counter()
    wall = wall1 - wall0
    clocks = sampler.stop(window=(t0_wall, time.time()))
    status = last.check()
    last.free()
    if status != ep.EP_OK:
        raise SystemExit("device error: %s" % ep.status_str(status))

    # Host cost of issuing one step through the binding, measured with the GPU
    # kept busy (no launch-queue back-pressure): the time a caller's CPU spends.
    host = []
    for _ in range(10):
        torch.cuda._sleep(20 * GPU_LEAD_CYCLES)
        t_issue = time.perf_counter()
        h = step()
        host.append(time.perf_counter() - t_issue)
        torch.cuda.synchronize()
        h.free()
    host_s = statistics.median(host)

    stp = [e[0].elapsed_time(e[1]) for e in events]

    # Attribution pass: the same K steps with a window around each call, for
    # the per-kernel times and the roofline (events between the calls keep the
    # kernels from overlapping, so these windows add up to a bit more than
    # the timed step).
    attr = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    last = None
    for i in range(args.steps):
        flush_l2()
        h = step(attr[i])
        if last is not None:
            last.free()
        last = h
    torch.cuda.synchronize()
    # Combine alone, with a clean L2 (flushed and drained before each call):
    # its in-step window also pays for writing back the dispatch's last dirty
    # L2 lines, a fixed amount (about the L2 size) whatever the batch.
    alone = []
    for i in range(args.steps):
        flush_l2()
        torch.cuda._sleep(GPU_LEAD_CYCLES // 2)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ep.ep_combine(last, y, tw, out)
        e1.record(stream)
        alone.append((e0, e1))
    torch.cuda.synchronize()
    com_alone_ms = reduce_max(sum(a.elapsed_time(b) for a, b in alone) / len(alone), world)
    last.free()
    lay = [e[0].elapsed_time(e[1]) for e in attr]
    dis = [e[1].elapsed_time(e[2]) for e in attr]
    com = [e[2].elapsed_time(e[3]) for e in attr]
    mean = lambda v: sum(v) / len(v)  # noqa: E731
    value, step_ms = job_throughput(mean(stp), nbytes["step"], args.steps, world)
    lay_ms, dis_ms, com_ms = (reduce_max(mean(v), world) for v in (lay, dis, com))

    peaks = measured_peaks()
    peak = peaks["hbm_gbs"]
    kern = {
        "note": "per-call windows from an attribution pass of the same steps",
        "layout": {"us": lay_ms * 1e3, "bytes": nbytes["layout"], "launches_per_step": layout_kernels,
                   "share_of_step_us": (step_ms - dis_ms - com_ms) * 1e3,
                   "share_note": "step minus the dispatch and combine windows: what the layout adds to a "
                                 "step with no events between its kernels"},
        "dispatch": {"us": dis_ms * 1e3, "bytes": nbytes["dispatch"],
                     "gbs": nbytes["dispatch"] / (dis_ms / 1e3) / 1e9},
        "combine": {"us": com_ms * 1e3, "bytes": nbytes["combine"],
                    "gbs": nbytes["combine"] / (com_ms / 1e3) / 1e9},
    }
    kern["combine_clean_l2"] = {"us": com_alone_ms * 1e3, "bytes": nbytes["combine"],
                                "gbs": nbytes["combine"] / (com_alone_ms / 1e3) / 1e9,
                                "note": "combine alone after an L2 flush (no dirty lines of the dispatch left)"}
    for kname in ("dispatch", "combine", "combine_clean_l2"):
        kern[kname]["frac_of_peak"] = kern[kname]["gbs"] / peak
        kern[kname]["frac_of_8tbs_nominal"] = kern[kname]["gbs"] / 8000.0
    dom = "combine" if com_ms >= dis_ms else "dispatch"
    src_file = {"combine": "combine.cu", "dispatch": "dispatch.cu"}[dom]
    tr = NCU_TRAFFIC.get((w.name, dom))
    traffic = tr["bytes"] if tr and tr["sha"] == source_sha(src_file) else None
    roofline = {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["gbs"], "peak": peak,
                "unit": "GB/s", "frac": kern[dom]["gbs"] / peak, "traffic": traffic,
                "algorithmic_bytes": nbytes[dom], "peak_source": peaks["source"]}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, dev, ep, x_cpu, idx_cpu, tw_cpu, y, nbytes, world)

    decode = None
    if not args.no_decode:
        decode = run_decode_latency(dev, ep)

    backward = None
    if not args.no_backward:
        backward = run_backward(w, dev, ep, idx, tw, y, flush_l2)

    gemm_layout = None
    if not args.no_gemm_layout:
        gemm_layout = run_gemm_layout(w, dev, ep, idx, x, flush_l2, y=y, tw=tw)

    overlap = None
    if not args.no_overlap:
        overlap = run_overlap(w, dev, ep, idx, x, tw, y, flush_l2)

    ranks = None
    if world == 1 and not args.no_ranks:
        ranks = run_ranks_emulated(w, dev, ep, flush_l2)

    ep_gpus = None
    if args.ep:
        ep_gpus = run_ep_across_gpus(args, w, world, rank, local)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, seed)

    if rank == 0:
        line = {
            "metric": "dispatch/combine HBM GB/s & % of peak; us/call at 8192 tok, H=7168, top-8",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": storage_dtype(w), "data": "synthetic",
            "config": workload_config(w, world),
            "kernels": kern, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "decode": decode, "backward": backward, "gemm_layout": gemm_layout, "overlap": overlap,
            "ranks_emulated": ranks,
            "ep_across_gpus": ep_gpus,
            "gpu_launches": launches, "clocks": clocks, "wall_s": wall,
            "host_us_per_step": host_s * 1e6,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_decode_latency(dev, ep, steps: int = 100) -> dict:
    """Decoding with a cached handle: one layout, then `steps` dispatch +
    combine calls with new x every step (x for step s drawn from seed
    1000 + s, staged in device memory beforehand, as a previous layer would
    leave it).  Reports us per call with plain launches and us per step for
    a replayed CUDA graph of dispatch + combine."""
    w = W.WORKLOADS["decode"]
    _, idx, tw = W.make_routing(w)
    res = ep.ep_layout(idx.to(dev), w.E, w.R, w.align, w.capacity)
    h = res.handle
    rows = h.num_recv_rows
    xs = torch.stack([W.make_x(w, 1000 + s) for s in range(steps)]).to(dev)
    xb = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    recv = torch.empty(rows, w.H, dtype=torch.float8_e4m3fn, device=dev)
    sc = torch.empty(rows, w.H // 128, dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev).manual_seed(21)
    y = torch.randn(rows, w.H, generator=g, device=dev).to(torch.bfloat16)
    twd = tw.to(dev)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ep.ep_dispatch(h, xb, True, recv, sc)
        ep.ep_combine(h, y, twd, out)

    for s in range(3):
        xb.copy_(xs[s])
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for s in range(steps):
        xb.copy_(xs[s])
        torch.cuda._sleep(GPU_LEAD_CYCLES // 4)
        ev[s][0].record(stream)
        ep.ep_dispatch(h, xb, True, recv, sc)
        ev[s][1].record(stream)
        ep.ep_combine(h, y, twd, out)
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    d_us = statistics.mean(e[0].elapsed_time(e[1]) for e in ev) * 1e3
    c_us = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) * 1e3

    # Back to back: `steps` launches of one call inside one event pair, so the
    # launch and event overheads of a single bracketed call drop out and what
    # is left is the GPU time per launch (each kernel still waits for its
    # predecessor; programmatic launch overlaps only the launch latency).
    def back_to_back(fn):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda._sleep(GPU_LEAD_CYCLES * 12)   # ~6 ms: the host queues every launch first
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / steps

    d_b2b = back_to_back(lambda: ep.ep_dispatch(h, xb, True, recv, sc))
    c_b2b = back_to_back(lambda: ep.ep_combine(h, y, twd, out))
    s_b2b = back_to_back(step)

    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        step()
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        step()
    for s in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    total = 0.0
    for s in range(steps):
        xb.copy_(xs[s])
        torch.cuda._sleep(GPU_LEAD_CYCLES // 4)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    g_b2b = back_to_back(graph.replay)
    status = h.check()
    del graph
    h.free()
    if status != ep.EP_OK:
        raise SystemExit("decode: device error %s" % ep.status_str(status))
    V = w.T * w.k
    disp_bytes = w.T * w.H * 2 + w.T * w.k * 4 + V * w.H + V * (w.H // 128) * 4
    comb_bytes = V * w.H * 2 + w.T * w.k * 8 + w.T * w.H * 2
    return {"workload": "decode", "tokens": w.T, "hidden": w.H, "topk": w.k, "experts": w.E,
            "capacity": w.capacity, "steps": steps, "dispatch_us": d_us, "combine_us": c_us,
            "step_us_plain": d_us + c_us, "step_us_graph": total / steps * 1e3,
            "dispatch_us_back_to_back": d_b2b, "combine_us_back_to_back": c_b2b,
            "step_us_back_to_back": s_b2b, "step_us_graph_back_to_back": g_b2b,
            "dispatch_bytes": disp_bytes, "combine_bytes": comb_bytes}


def run_backward(w, dev, ep, idx_dev, tw_dev, y_dev, flush_l2, steps: int = 20) -> dict:
    """The backward pair on the step's layout: ep_dispatch_backward (the
    combine with unit weights) and ep_combine_backward (weighted scatter of
    grad_out plus the grad_weights dot products), each timed with the L2
    flushed before every call."""
    T, H, k = w.T, w.H, w.k
    res = ep.ep_layout(idx_dev, w.E, w.R, w.align, w.capacity)
    h = res.handle
    rows = h.num_recv_rows
    g = torch.Generator(device=dev).manual_seed(77)
    grad_recv = torch.randn(rows, H, generator=g, device=dev).to(torch.bfloat16)
    grad_out = torch.randn(T, H, generator=g, device=dev).to(torch.bfloat16)
    grad_x = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    grad_y = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
    grad_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        ts = []
        for i in range(steps + 3):
            flush_l2()
            torch.cuda._sleep(GPU_LEAD_CYCLES // 2)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= 3:
                ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ts) * 1e3

    d_us = timed(lambda: ep.ep_dispatch_backward(h, grad_recv, grad_x))
    c_us = timed(lambda: ep.ep_combine_backward(h, grad_out, tw_dev, y=y_dev, grad_y=grad_y,
                                                grad_weights=grad_w))
    # per-row routing outputs (recv_topk_idx / recv_topk_weights / slot), which
    # a weighted expert GEMM or a per-row backward reads
    t_us = timed(lambda: ep.ep_dispatch_topk(h, tw_dev))
    status = h.check()
    h.free()
    if status != ep.EP_OK:
        raise SystemExit("backward: device error %s" % ep.status_str(status))
    V = int((idx_dev >= 0).sum().item())
    d_bytes = V * H * 2 + T * k * 4 + T * H * 2
    c_bytes = T * H * 2 + V * H * 2 + T * k * 8 + V * H * 2 + T * k * 4
    t_bytes = rows * 4 + T * k * 4 + V * 4 + (w.E + 1) * 4 + rows * 12
    return {"dispatch_backward": {"us": d_us, "bytes": d_bytes, "gbs": d_bytes / d_us / 1e3},
            "combine_backward": {"us": c_us, "bytes": c_bytes, "gbs": c_bytes / c_us / 1e3},
            "dispatch_topk": {"us": t_us, "bytes": t_bytes, "note": "latency-bound (~1.6 MB)"}}


def run_gemm_layout(w, dev, ep, idx_dev, x_dev, flush_l2, steps: int = 20, y=None, tw=None) -> dict | None:
    """The FP8 dispatch options that serve grouped expert GEMMs, on the
    step's layout, each timed with the L2 flushed before every call: scales
    row-major [rows, H/128] (the step's form); column-major [H/128, ld]
    (ld = rows rounded up to 4) through the per-token table and column fill
    (ep_dispatch_fp8_colmajor) and, for comparison, with one scattered store
    per row and group (ep_dispatch_ex); pre-quantised input (e4m3 codes +
    scales, copied unchanged) with row-major and column-major scales.

    With y and tw, also each of the two quantising forms followed by the
    step's combine in one window (`in_step`): a dispatch leaves L2 full of
    dirty lines whose write-back the next kernel pays for, and the column
    fill, run right after the dispatch, pays part of that inside its own
    window; the difference of the two windows is what the column-major
    form adds to a step."""
    if not w.fp8:
        return None
    T, H, k = w.T, w.H, w.k
    G = H // 128
    res = ep.ep_layout(idx_dev, w.E, w.R, w.align, w.capacity)
    h = res.handle
    rows = h.num_recv_rows
    ld = (rows + 3) // 4 * 4
    recv = torch.empty(rows, H, dtype=torch.float8_e4m3fn, device=dev)
    sc_row = torch.empty(rows, G, dtype=torch.float32, device=dev)
    sc_col = torch.empty(G, ld, dtype=torch.float32, device=dev)
    # pre-quantised input (plumbing, outside the timed calls): per-group scales and codes
    xf = x_dev.float().view(T, G, 128)
    amax = xf.abs().amax(-1).clamp_min(1e-30)
    xs = (amax / 448.0).contiguous()
    xq = (xf * (448.0 / amax)[..., None]).view(T, H).to(torch.float8_e4m3fn).contiguous()
    del xf
    stream = torch.cuda.current_stream()

    def timed(fn):
        ts = []
        for i in range(steps + 3):
            flush_l2()
            torch.cuda._sleep(GPU_LEAD_CYCLES // 2)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= 3:
                ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ts) * 1e3

    row_us = timed(lambda: ep.ep_dispatch_ex(h, x_dev, True, recv_x=recv, recv_scales=sc_row))
    col_us = timed(lambda: ep.ep_dispatch_ex(h, x_dev, True, recv_x=recv, recv_scales=sc_col, scale_layout="col"))
    tok = torch.empty(T, G, dtype=torch.float32, device=dev)
    colt_us = timed(lambda: ep.ep_dispatch_fp8_colmajor(h, x_dev, recv_x=recv, recv_scales=sc_col, token_scales=tok))
    pq_us = timed(lambda: ep.ep_dispatch_ex(h, xq, True, x_scales=xs, recv_x=recv, recv_scales=sc_row))
    pqc_us = timed(lambda: ep.ep_dispatch_ex(h, xq, True, x_scales=xs, recv_x=recv, recv_scales=sc_col,
                                             scale_layout="col"))
    in_step = None
    if y is not None and tw is not None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        row_c = timed(lambda: (ep.ep_dispatch_ex(h, x_dev, True, recv_x=recv, recv_scales=sc_row),
                               ep.ep_combine(h, y, tw, out)))
        col_c = timed(lambda: (ep.ep_dispatch_fp8_colmajor(h, x_dev, recv_x=recv, recv_scales=sc_col,
                                                           token_scales=tok),
                               ep.ep_combine(h, y, tw, out)))
        in_step = {"row_major_then_combine_us": row_c, "column_major_then_combine_us": col_c,
                   "column_major_adds_us": col_c - row_c,
                   "column_major_equivalent_us": row_us + col_c - row_c}
    status = h.check()
    h.free()
    if status != ep.EP_OK:
        raise SystemExit("gemm layout: device error %s" % ep.status_str(status))
    V = int((idx_dev >= 0).sum().item())
    q_bytes = T * H * 2 + T * k * 4 + V * H + V * G * 4
    pq_bytes = T * H + T * G * 4 + T * k * 4 + V * H + V * G * 4
    return {"scales_row_major": {"us": row_us, "bytes": q_bytes, "gbs": q_bytes / row_us / 1e3},
            "scales_column_major_scattered": {"us": col_us, "bytes": q_bytes, "gbs": q_bytes / col_us / 1e3,
                                              "ld": ld, "call": "ep_dispatch_ex"},
            "scales_column_major": {"us": colt_us, "bytes": q_bytes, "gbs": q_bytes / colt_us / 1e3, "ld": ld,
                                    "call": "ep_dispatch_fp8_colmajor (per-token table + column fill)",
                                    "table_bytes": T * G * 4},
            "prequantised_input": {"us": pq_us, "bytes": pq_bytes, "gbs": pq_bytes / pq_us / 1e3},
            "prequantised_input_column_major": {"us": pqc_us, "bytes": pq_bytes, "gbs": pq_bytes / pqc_us / 1e3,
                                                "ld": ld},
            "in_step": None if in_step is None else dict(
                in_step, column_major_equivalent_gbs=q_bytes / in_step["column_major_equivalent_us"] / 1e3)}


def run_ranks_emulated(w, dev, ep, flush_l2, worlds=(1, 8), steps: int = 10) -> dict:
    """Expert parallelism across W ranks, every rank emulated on this GPU:
    the workload split into W source batches of T/W tokens, each rank's plan,
    then every rank's peer dispatch and peer combine (each rank's kernels in
    turn on one stream, all buffers in this GPU's HBM).  W = 1 runs the whole
    batch through the peer-addressed kernels (compare with the local ones:
    the cost of the indirection); W = 8 gives the plan's latency at eight
    ranks and eight back-to-back launches of T/8 tokens.  Not NVLink, which
    needs GPUs."""
    stream = torch.cuda.current_stream()

    def timed(fn):
        ts = []
        for i in range(steps + 3):
            flush_l2()
            torch.cuda._sleep(GPU_LEAD_CYCLES)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= 3:
                ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ts) * 1e3

    out = {"note": "all ranks emulated on one GPU: every store and load is local HBM, no NVLink"}
    for world in worlds:
        Tr = w.T // world
        parts = [W.make_routing(w.scaled(T=Tr), seed=7000 + r) for r in range(world)] if world > 1 else \
            [W.make_routing(w, seed=0)]
        rows = ep.ep_peer_max_recv_rows(Tr * world, w.k, w.E, world)
        rdt = torch.float8_e4m3fn if w.fp8 else torch.bfloat16
        recv = [torch.empty(rows, w.H, dtype=rdt, device=dev) for _ in range(world)]
        sc = [torch.empty(rows, w.H // 128, dtype=torch.float32, device=dev) for _ in range(world)] \
            if w.fp8 else None
        g = torch.Generator(device=dev).manual_seed(99)
        ys = [torch.randn(rows, w.H, generator=g, device=dev).to(torch.bfloat16) for _ in range(world)]
        peers = ep.Peers(world, recv, sc, ys, rows)
        xs = [p[0].to(dev) for p in parts]
        idxs = [p[1].to(dev) for p in parts]
        tws = [p[2].to(dev) for p in parts]
        lays = [ep.ep_layout(i, w.E, world) for i in idxs]
        counts = torch.stack([l.num_tokens_per_expert for l in lays])
        plans = [ep.ep_plan_create(l.handle, i, counts, r, world, rows)
                 for r, (l, i) in enumerate(zip(lays, idxs))]
        plan_us = timed(lambda: ep.ep_plan_create(lays[0].handle, idxs[0], counts, 0, world, rows).free())
        d_us = timed(lambda: [ep.ep_dispatch_peer(plans[r], peers, xs[r], w.fp8) for r in range(world)])
        c_us = timed(lambda: [ep.ep_combine_peer(plans[r], peers, tws[r], w.H) for r in range(world)])
        if any(p.check() != ep.EP_OK for p in plans):
            raise SystemExit("ranks_emulated: plan error")
        V = sum(int((p[1] >= 0).sum()) for p in parts)
        T = Tr * world
        if w.fp8:
            d_bytes = T * w.H * 2 + V * w.H + V * (w.H // 128) * 4 + T * w.k * 8
        else:
            d_bytes = T * w.H * 2 + V * w.H * 2 + T * w.k * 8
        c_bytes = V * w.H * 2 + T * w.k * 12 + T * w.H * 2
        out["world_%d" % world] = {
            "tokens_per_rank": Tr, "plan_us": plan_us,
            "dispatch": {"us": d_us, "bytes": d_bytes, "gbs": d_bytes / d_us / 1e3},
            "combine": {"us": c_us, "bytes": c_bytes, "gbs": c_bytes / c_us / 1e3},
            "recv_rows_per_rank": [p.recv_rows_host() for p in plans]}
        for p in plans:
            p.free()
        for l in lays:
            l.handle.free()
        peers.free()
        del recv, sc, ys
        torch.cuda.empty_cache()
    return out


# Assumed NVLink peer bandwidth per direction per GPU for the floor of the
# cross-GPU step: a figure quoted for this GPU type's peer copies, not
# measured by this repository (no run here has had two GPUs).  900 GB/s is
# the nominal NVLink 5 figure.
NVLINK_PEER_GBS = 770.0


def run_ep_across_gpus(args, w, world, rank, local, steps: int = 10) -> dict:
    """Expert parallelism across the job's GPUs (opt-in, --ep).  Every rank
    holds its own batch of the workload's T tokens, the E experts are split
    over the W ranks, and a step is the multi-GPU protocol of EpGroup: local
    layout, count all-gather and plan; dispatch by peer stores into the
    owners' receive buffers; combine by peer loads from the owners' expert
    outputs; NCCL collectives between.  Device time per step is the max over
    ranks.  NVLink bytes are the rows (plus FP8 scales) whose owner is another
    rank, each way; with W = 1 every row is local."""
    import socket
    import torch.distributed as dist
    from combine_ep_layout_10_b200 import ep, group
    created = False
    if not dist.is_initialized():
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        with _StdoutToStderr():
            dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        created = True
    dev = torch.device("cuda", local)
    x_cpu, idx_cpu, tw_cpu = W.make_routing(w, replica_seed(args.seed, rank))
    x, idx, tw = x_cpu.to(dev), idx_cpu.to(dev), tw_cpu.to(dev)
    rows = ep.ep_peer_max_recv_rows(world * w.T, w.k, w.E, world)
    g = group.EpGroup(w.E, w.H, rows, fp8=w.fp8)
    gen = torch.Generator(device=dev).manual_seed(31 + rank)
    g.y.copy_(torch.randn(rows, w.H, generator=gen, device=dev).to(torch.bfloat16))
    for _ in range(max(args.warmup, 1)):
        plan = g.dispatch(x, idx)
        g.combine(plan, tw)
        plan.free()
    torch.cuda.synchronize(dev)
    dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    plans = []
    e0.record()
    for _ in range(steps):
        plan = g.dispatch(x, idx)
        g.combine(plan, tw)
        plans.append(plan)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = reduce_max(e0.elapsed_time(e1) / steps, world)
    d = plans[0].export()["dst"]
    owner = d[..., 0]
    remote = int(((owner >= 0) & (owner != rank)).sum().item())     # rows this rank sends away
    own = int((owner == rank).sum().item())                          # rows it keeps
    recv = plans[0].recv_rows_host()
    if any(p.check() != ep.EP_OK for p in plans):
        raise SystemExit("ep_across_gpus: plan error")
    for p in plans:
        p.free()
    g.close()
    if created:
        dist.destroy_process_group()
    row_d = w.H * (1 if w.fp8 else 2) + (w.H // 128 * 4 if w.fp8 else 0)
    row_c = w.H * 2
    inbound = recv - own                                             # rows other ranks send here
    # dispatch: out = rows sent, in = rows received; combine: the reverse, at bf16 width
    d_link = reduce_max(float(max(remote, inbound) * row_d), world)
    c_link = reduce_max(float(max(remote, inbound) * row_c), world)
    floor_ms = (d_link + c_link) / (NVLINK_PEER_GBS * 1e9) * 1e3
    return {"world": world, "tokens_per_rank": w.T, "ms_per_step": ms,
            "rows_sent_this_rank": remote, "rows_received_from_peers_this_rank": inbound,
            "nvlink_bytes_dispatch_busiest_rank": d_link, "nvlink_bytes_combine_busiest_rank": c_link,
            "nvlink_floor_ms": floor_ms,
            "frac_of_nvlink_floor": (floor_ms / ms) if ms > 0 and floor_ms > 0 else None,
            "note": "per step: layout + all-gather + plan, peer dispatch, peer combine; floor = the "
                    "busiest rank's larger direction per phase at an assumed 770 GB/s peer bandwidth (not measured here)"}


def run_overlap(w, dev, ep, idx_dev, x_dev, tw_dev, y_dev, flush_l2, reps: int = 10) -> dict:
    """SM-budgeted communication overlapped with compute: a bf16 GEMM of the
    expert-GEMM shape [T, H] x [H, 4096] (cuBLAS, the stand-in for the work
    the budget leaves SMs to) on the current stream, and dispatch + combine
    with num_sms = n on a second stream.  Reports each alone and both
    together (device time from the first launch to the last completion)."""
    res = ep.ep_layout(idx_dev, w.E, w.R, w.align, w.capacity)
    h = res.handle
    rows = h.num_recv_rows
    rdt = torch.float8_e4m3fn if w.fp8 else torch.bfloat16
    recv = torch.empty(rows, w.H, dtype=rdt, device=dev)
    sc = torch.empty(rows, w.H // 128, dtype=torch.float32, device=dev) if w.fp8 else None
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    g = torch.Generator(device=dev).manual_seed(3)
    wt = torch.randn(w.H, 4096, generator=g, device=dev).to(torch.bfloat16)
    act = torch.randn(w.T, w.H, generator=g, device=dev).to(torch.bfloat16)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side_hi = torch.cuda.Stream(priority=-1)  # high priority: scheduled first as SMs free up

    def comm(n):
        ep.ep_dispatch_ex(h, x_dev, w.fp8, recv_x=recv, recv_scales=sc, num_sms=n)
        ep.ep_combine_ex(h, y_dev, tw_dev, out=out, num_sms=n)

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            flush_l2()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(GPU_LEAD_CYCLES // 2)
            e0.record(main)
            fn()
            e1.record(main)
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.mean(ts)

    def gemm():
        torch.matmul(act, wt)

    def both(n, stream):
        stream.wait_stream(main)
        with torch.cuda.stream(stream):
            comm(n)
        gemm()
        main.wait_stream(stream)

    out_d = {"gemm_us": timed(gemm)}
    for n in (16, 32, 64, 0):
        key = "all" if n == 0 else str(n)
        out_d["comm_us_sms_" + key] = timed(lambda: comm(n))
        out_d["both_us_sms_" + key] = timed(lambda: both(n, side))
        out_d["both_hiprio_us_sms_" + key] = timed(lambda: both(n, side_hi))
    h.free()
    return out_d


def run_e2e(args, w, dev, ep, x_cpu, idx_cpu, tw_cpu, y_dev, nbytes, world):
    """Same step through the public API from pinned host buffers: H2D of x,
    topk_idx, topk_w and the expert outputs y, the three calls, D2H of out --
    every step's copies inside the timed region.  Steps are pipelined two
    deep, as a serving loop would run them: step n+1's uploads (one copy
    stream) overlap step n's kernels (the compute stream) and step n-1's
    readback (a second copy stream, the other PCIe direction); events order
    each buffer set's reuse."""
    T, H, E, R = w.T, w.H, w.E, w.R
    xh = x_cpu.pin_memory()
    ih = idx_cpu.pin_memory()
    th = tw_cpu.pin_memory()
    yh = y_dev.cpu().pin_memory()
    ohs = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    rdt = torch.float8_e4m3fn if w.fp8 else torch.bfloat16
    rows = yh.shape[0]
    sets = []
    for _ in range(2):
        sets.append({"x": torch.empty_like(xh, device=dev), "idx": torch.empty_like(ih, device=dev),
                     "tw": torch.empty_like(th, device=dev), "y": torch.empty_like(yh, device=dev),
                     "recv": torch.empty(rows, H, dtype=rdt, device=dev),
                     "scales": torch.empty(rows, H // 128, dtype=torch.float32, device=dev) if w.fp8 else None,
                     "out": torch.empty(T, H, dtype=torch.bfloat16, device=dev)})
    h2d = sum(t.numel() * t.element_size() for t in (xh, ih, th, yh))
    d2h = ohs[0].numel() * ohs[0].element_size()
    comp = torch.cuda.current_stream()
    cin = torch.cuda.Stream(device=dev)
    cout = torch.cuda.Stream(device=dev)

    def run(n_steps):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, comp_done, out_done = [], [], []
        handles = []
        for s in range(n_steps):
            b = sets[s % 2]
            with torch.cuda.stream(cin):
                if s >= 2:
                    cin.wait_event(comp_done[s - 2])      # set b no longer read by step s-2
                b["x"].copy_(xh, non_blocking=True)
                b["idx"].copy_(ih, non_blocking=True)
                b["tw"].copy_(th, non_blocking=True)
                b["y"].copy_(yh, non_blocking=True)
                e = ev(); e.record(cin); in_ready.append(e)
            comp.wait_event(in_ready[s])
            if s >= 2:
                comp.wait_event(out_done[s - 2])          # out of set b read back
            res = ep.ep_layout(b["idx"], E, R, w.align, w.capacity)
            ep.ep_dispatch(res.handle, b["x"], w.fp8, b["recv"], b["scales"])
            ep.ep_combine(res.handle, b["y"], b["tw"], b["out"])
            handles.append(res.handle)
            e = ev(); e.record(comp); comp_done.append(e)
            with torch.cuda.stream(cout):
                cout.wait_event(comp_done[s])
                ohs[s % 2].copy_(b["out"], non_blocking=True)
                e = ev(); e.record(cout); out_done.append(e)
        comp.wait_event(out_done[-1])
        return handles

    n_steps = max(3, min(args.steps, 10))
    for h in run(2):
        h.free()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    cin.wait_event(e0)
    handles = run(n_steps)
    e1.record(comp)
    torch.cuda.synchronize()
    for h in handles:
        h.free()
    ms = reduce_max(e0.elapsed_time(e1) / n_steps, world)
    total = reduce_sum(nbytes["step"], world)
    # The link this number is bound by: one plain pinned upload of the same
    # bytes (the largest input), timed alone on the copy stream.
    big = sets[0]["y"]
    up = []
    for _ in range(3):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(cin)
        big.copy_(yh, non_blocking=True)
        b.record(cin)
        torch.cuda.synchronize()
        up.append(a.elapsed_time(b))
    h2d_gbs = yh.numel() * yh.element_size() / (min(up) / 1e3) / 1e9
    step_h2d_gbs = h2d / (ms / 1e3) / 1e9
    return {"value": total / (ms / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_steps,
            "pipelined": "2 deep: uploads, kernels and readback of neighbouring steps overlap",
            "roofline": {"bound": "pcie_h2d", "achieved": step_h2d_gbs, "peak": h2d_gbs, "unit": "GB/s",
                         "frac": step_h2d_gbs / h2d_gbs,
                         "peak_source": "one pinned %.0f MB upload timed alone" % (yh.numel() * yh.element_size() / 1e6)}}


def main():
    args = parse()
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
