#!/usr/bin/env python
"""Benchmark of the routed int4 MoE layer (libcolimoe) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--tokens T] [--path auto|gemv|gemm|fused] [--impl own|reference]

A step is one forward of the layer (router, union, int4 experts, SwiGLU, combine)
over one batch of synthetic tokens already resident in HBM.  Between timed steps
a 256 MiB buffer is written to flush L2 (126 MB); each step is timed alone with
CUDA events on the launching stream, so the flushes are not counted.  Under
torchrun every rank runs an independent replica (the layer does not shard here);
the job time is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at batch 1-512; int4 weight GB/s as % of B200 HBM peak"
UNIT = "tokens/s"
SPEC_HBM_GBS = 8000.0  # the B200's nominal HBM3e bandwidth (~8 TB/s), beside the measured copy peak


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clock sampling during the timed region (NVML, ~2 ms period)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, dev_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def profiled_traffic(kernel_src: str, profile: str, profiles_dir: str | None = None):
    """DRAM bytes per launch (read + write) from the ncu summary in profiles/,
    valid only while the kernel source still has the hash the capture names."""
    import hashlib
    try:
        text = open(os.path.join(profiles_dir or os.path.join(ROOT, "profiles"), profile)).read()
        digest = hashlib.sha256(open(os.path.join(ROOT, kernel_src), "rb").read()).hexdigest()
    except OSError:
        return None
    want = traffic = None
    for line in text.splitlines():
        if "sha256 prefix" in line:
            want = line.split("sha256 prefix")[1].split()[0]
        if line.startswith("| traffic_bytes_per_launch |"):
            traffic = float(line.split("|")[2])
    return traffic if want and digest.startswith(want) else None


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def path_ids():
    import int4_routed_expert_top_b200 as cm
    return {"auto": cm.COLI_PATH_AUTO, "gemv": cm.COLI_PATH_GEMV, "gemm": cm.COLI_PATH_GEMM,
            "fused": cm.COLI_PATH_FUSED, "twopass": cm.COLI_PATH_TWOPASS}


def resolve_path(wl, T, path_name, bits=4):
    """The path a forward takes (AUTO resolved as include/coli_moe.h states)."""
    if path_name != "auto":
        return path_name
    if (T <= 64 and T * (wl.k + wl.n_shared) <= 640 and wl.E <= 256 and wl.k <= 32
            and wl.n_shared <= 4 and wl.H % 256 == 0 and wl.I <= 4096):
        return "fused"
    if (bits == 4 and 64 < T <= 1024 and wl.E <= 256 and wl.n_shared <= 4
            and wl.H % 256 == 0 and wl.I % 256 == 0):
        return "twopass"
    return "gemv" if T < 48 else "gemm"


def launches_per_layer(wl, T, path_name, fused):
    """This library's kernel launches in one forward of one layer."""
    path_name = resolve_path(wl, T, path_name)
    if fused or path_name == "fused":
        return 3                                  # router, fused kernel, combine
    select = 1 if T * wl.E <= 4096 and T <= 128 else 2   # top-k and union together or apart
    if path_name == "twopass":
        # router, select, x records, gate/up pass, h records, down pass, combine
        return 1 + select + 5
    if path_name == "gemv":
        return 1 + select + 2                     # router, select, gate/up GEMV, down GEMV
    # router (+ the fp16 activation operand past 64 tokens), select, gather,
    # GEMM, h, GEMM, combine
    return (2 if T > 64 else 1) + select + 5


def workload(name):
    import synth
    return synth.WORKLOADS[name]


def token_pool(wl, T, n_batches, rank, device):
    import synth
    import torch
    xs = [synth.tokens(wl, T, layer=0, step=rank * n_batches + i) for i in range(n_batches)]
    x = torch.stack(xs).to(device)
    if wl.x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x.contiguous()


def build_layers(wl, device, bits=4):
    import synth
    from int4_routed_expert_top_b200.device_layer import DeviceLayer
    layers = []
    for l in range(wl.layers):
        wr, b = synth.router(wl, l)
        mats = (synth.T_GATE, synth.T_UP, synth.T_DOWN)
        layers.append(DeviceLayer(
            wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, wr, b,
            expert_masters=lambda e, l=l: tuple(synth.expert_master(wl, l, t, e, device=device)
                                                for t in mats),
            routed_scale=wl.routed_scale, norm_topk=wl.norm_topk, device=device, bits=bits))
    return layers


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------
class OracleSampler:
    """The oracle, as it stands, on whole tokens of the workload: routing on the
    full router, dequantisation of every expert matrix the token uses, the SwiGLU
    experts and the combine.  Building the container (quantisation) is offline
    work and is not timed."""

    def __init__(self, wl):
        import synth
        import torch
        self.wl = wl
        self.dev = "cuda" if torch.cuda.is_available() else "cpu"
        wr, b = synth.router(wl, 0)
        self.wr, self.b = wr.numpy(), b.numpy()
        self.x = synth.tokens(wl, max(wl.T, 64), layer=0, step=0).numpy()
        self.cont = {}
        self.done = 0

    def _container(self, e):
        import oracle
        import synth
        if e not in self.cont:
            self.cont[e] = []
            for t in (synth.T_GATE, synth.T_UP, synth.T_DOWN):
                m = synth.expert_master(self.wl, 0, t, e, device=self.dev).cpu().numpy()
                self.cont[e].append((oracle.quantize(m, self.wl.group), m.shape[1]))
        return self.cont[e]

    def step(self) -> float:
        """One token through the oracle; returns its CPU seconds."""
        import oracle
        wl, t = self.wl, self.done % self.x.shape[0]
        idx, w, _ = oracle.route(self.x[t:t + 1], self.wr, self.b, wl.k, wl.routed_scale,
                                 wl.norm_topk)
        ids = [int(e) for e in idx[0]] + [wl.E + s for s in range(wl.n_shared)]
        for e in ids:
            self._container(e)
        t0 = time.perf_counter()
        idx, w, _ = oracle.route(self.x[t:t + 1], self.wr, self.b, wl.k, wl.routed_scale,
                                 wl.norm_topk)
        ex = [tuple(oracle.dequantize(p, s, K, wl.group) for (p, s), K in self._container(e))
              for e in ids]
        oracle.token_forward(self.x[t], w[0], ex, wl.n_shared)
        self.done += 1
        return time.perf_counter() - t0


def host_cpu():
    """The host the CPU baseline ran on: logical CPUs, the ones this process may
    use, and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    aff = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else None
    return {"nproc": os.cpu_count(), "affinity": aff, "cpu_model": model}


def oracle_sample(wl, budget_s=12.0):
    smp = OracleSampler(wl)
    spent, n = 0.0, 0
    while n == 0 or spent < budget_s:
        spent += smp.step()
        n += 1
    return n / spent, n, spent, smp


def oracle_threads():
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return max(1, min(16, n or 1))


def oracle_sample_parallel(smp, threads, budget_s=10.0):
    """The same oracle steps on `threads` host threads at once (ctypes releases
    the interpreter lock inside the oracle, so each thread runs on its own
    core), over the tokens the single-threaded sample prepared: parallel over
    tokens, as the oracle's own OpenMP loop over tokens is.  Returns tokens/s
    of wall time and the tokens done."""
    import concurrent.futures as cf
    n_tok = max(smp.done, 1)
    t0 = time.perf_counter()

    def worker(w):
        done, i = 0, w
        while time.perf_counter() - t0 < budget_s or done == 0:
            sub = OracleSampler.__new__(OracleSampler)
            sub.__dict__.update(smp.__dict__)
            sub.done = i % n_tok
            sub.step()
            done += 1
            i += threads
        return done

    with cf.ThreadPoolExecutor(threads) as ex:
        total = sum(ex.map(worker, range(threads)))
    wall = time.perf_counter() - t0
    return total / wall, total, wall


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(args.workload)
    per_step = []
    smp = OracleSampler(wl)
    t_all = time.perf_counter()
    for i in range(args.warmup + args.steps):
        if time.perf_counter() - t_all > 150 and len(per_step) >= 1:
            break                       # keep the reference arm within a few minutes
        secs = smp.step()
        if i >= args.warmup:
            per_step.append(secs)
    threads = oracle_threads()
    par_rate, par_n, par_s = oracle_sample_parallel(smp, threads, budget_s=20.0)
    tok_s = par_rate / wl.layers
    sample = (f"{par_n} steps of 1 token each (router over all {wl.E} experts, "
              f"dequantisation of the {wl.k}+{wl.n_shared} expert matrices it uses, SwiGLU, "
              f"combine) of workload {wl.name} on {threads} host threads at once "
              f"({par_s:.1f} s wall); single-threaded median step "
              f"{1e3 * statistics.median(per_step):.0f} ms over {len(per_step)} steps")
    if wl.layers > 1:
        sample += (f"; one layer per step, the rate divided by the {wl.layers} layers of the "
                   f"stack (every layer has the same shapes)")
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT,
            "n_gpus": args.gpus, "steps": len(per_step), "warmup": args.warmup,
            "ms_per_step": 1e3 / tok_s, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens_per_step": 1},
            "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample, "host": host_cpu(),
                             "single_thread": {"value": 1.0 / statistics.median(per_step)
                                               / wl.layers, "unit": UNIT, "cores": 1}},
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# job-wide numbers over ranks (one replica per GPU)
# ---------------------------------------------------------------------------
def max_over_ranks(ms: float, world: int, device) -> float:
    """Length of a timed region as the job sees it: the largest over the ranks
    (every rank calls this at the same point, so the collectives stay in step)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, job_ms: float) -> float:
    """Whole-job throughput: the tokens of every rank over the job's time."""
    return tokens_per_rank * world / (job_ms / 1e3)


# ---------------------------------------------------------------------------
# own arm
# ---------------------------------------------------------------------------
def run_ep(args):
    """Expert-parallel layer over N GPUs (one process each): every rank routes
    all tokens, computes the picks of its own experts and the ranks' partial
    outputs are summed by one NCCL all-reduce per step.  Strong scaling: the
    same T tokens per step whatever N.  Launched eagerly (no graph holds the
    collective); each step timed with CUDA events, the slowest rank's median."""
    import torch
    import torch.distributed as dist
    import int4_routed_expert_top_b200 as cm
    from int4_routed_expert_top_b200 import ep
    from int4_routed_expert_top_b200.device_layer import DeviceLayer
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = workload(args.workload)
    if wl.layers != 1:
        raise SystemExit("--ep times one layer")
    T = args.tokens or wl.T
    path = path_ids()[args.path]
    lo, hi = ep.expert_range(wl.E, rank, world)
    wr, b = synth.router(wl, 0)
    mats = (synth.T_GATE, synth.T_UP, synth.T_DOWN)
    L = DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, wr, b,
                    expert_masters=lambda e: tuple(synth.expert_master(wl, 0, t, e, device=dev)
                                                   for t in mats),
                    routed_scale=wl.routed_scale, norm_topk=wl.norm_topk, device=dev,
                    expert_range=(lo, hi) if world > 1 else None,
                    with_shared=rank == ep.SHARED_RANK)
    n_pool = 64 if T <= 16 else 2
    xpool = token_pool(wl, T, n_pool, 0, dev)          # the same tokens on every rank
    y = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    ws = L.workspace(T)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, x=None):
        cm.coli_moe_forward_ex(L.handle, xpool[i % n_pool] if x is None else x, T, y, ws,
                               path=path)
        if world > 1:
            ep.combine_partials(y)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush.zero_()
            starts[i].record(stream)
            step(i)
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    med = max_over_ranks(statistics.median(step_ms), world, dev)
    # end to end: pinned host tokens in, the summed y out, every step
    xh = torch.empty(xpool.shape, dtype=xpool.dtype, pin_memory=True)
    xh.copy_(xpool.cpu())
    yh = torch.empty((T, wl.H), dtype=torch.float32, pin_memory=True)
    xd = torch.empty_like(xpool[0])
    e2e = []
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        xd.copy_(xh[i % n_pool], non_blocking=True)
        step(i, xd)
        yh.copy_(y, non_blocking=True)
        s1.record(stream)
        e2e.append((s0, s1))
    torch.cuda.synchronize()
    barrier()
    e2e_med = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in e2e), world, dev)
    line = {"metric": METRIC, "value": T / (med / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": med, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded SplitMix64/Box-Muller, random-init weights)",
            "config": {"workload": wl.name, "tokens_per_step": T, "parallelism": f"ep{world}",
                       "experts_per_rank": hi - lo, "shared_on_rank": ep.SHARED_RANK,
                       "collective": "NCCL all-reduce (sum) of y [T, H] f32 per step",
                       "l2": "256 MiB buffer written between timed steps, not timed",
                       "launch": "eager (no graph)"},
            "clocks": clocks.summary(),
            "gpu_launches": launches_per_layer(wl, T, args.path, T <= 64) * K,
            "e2e": {"value": T / (e2e_med / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": int(xpool[0].numel() * xpool.element_size()),
                    "d2h_bytes_per_step": int(T * wl.H * 4)}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    L.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="glm_decode")
    ap.add_argument("--tokens", type=int, default=0, help="override tokens per step")
    ap.add_argument("--path", default="auto", choices=("auto", "gemv", "gemm", "fused", "twopass"))
    ap.add_argument("--impl", default="own", choices=("own", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="override routed experts (small-footprint profiling layers)")
    ap.add_argument("--bits", type=int, default=4, choices=(4, 8),
                    help="bits per expert weight code (8: the 8-bit container, fused path)")
    ap.add_argument("--topp", type=float, default=0.0,
                    help="adaptive expert top-p (0: every pick; coli_moe_layer_set_topp)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: each rank holds E/N routed experts (rank 0 the "
                         "shared ones), one all-reduce of y per step")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)
    if args.ep:
        return run_ep(args)

    import torch
    import torch.distributed as dist
    import int4_routed_expert_top_b200 as cm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = workload(args.workload)
    if args.experts:
        import dataclasses
        wl = dataclasses.replace(wl, E=args.experts)
    T = args.tokens or wl.T
    path = path_ids()[args.path]
    # the path AUTO resolves to (include/coli_moe.h)
    resolved = resolve_path(wl, T, args.path, args.bits)
    fused = resolved == "fused"
    layers = build_layers(wl, dev, args.bits)
    if args.topp:
        for l in layers:
            cm.coli_moe_layer_set_topp(l.handle, args.topp)
    L0 = layers[0]
    n_pool = 64 if T <= 16 else 2
    xpool = token_pool(wl, T, n_pool, rank, dev)
    y = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    xs = torch.empty((T, wl.H), dtype=torch.float32, device=dev)   # stack residual stream
    handles = [l.handle for l in layers]
    # one workspace for both the device-resident steps and the host-buffer calls
    # (which need the forward's workspace plus the staging of x and y)
    ws = torch.empty((cm.coli_moe_stack_host_workspace_size(handles, T) if wl.layers > 1
                      else cm.coli_moe_host_workspace_size(L0.handle, T),),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    idx_all = torch.empty((max(args.steps, n_pool), T, wl.k), dtype=torch.int32, device=dev)
    w_all = torch.empty((max(args.steps, n_pool), T, wl.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, events=None, record_idx=False):
        xi = xpool[i % n_pool]
        if wl.layers == 1:
            cm.coli_moe_forward_ex(L0.handle, xi, T, y, ws, path=path,
                                   idx_out=idx_all[i] if record_idx else None,
                                   w_out=w_all[i] if record_idx else None, events=events)
        else:
            xs.copy_(xi)
            cm.coli_moe_stack_forward([l.handle for l in layers], xs, T, wl.eps, ws, path=path)

    for i in range(args.warmup):
        flush.zero_()
        step(i, record_idx=i < args.steps)
    torch.cuda.synchronize()
    # routing of every pool slot (deterministic), for the weight-byte count
    for j in range(n_pool):
        step(j, record_idx=True)
    torch.cuda.synchronize()
    slot_idx = idx_all[:n_pool].cpu().numpy() if wl.layers == 1 else None
    # picks of weight 0 (dropped by top-p) are not computed: their experts are not read
    slot_w = w_all[:n_pool].cpu().numpy() if wl.layers == 1 else None

    # one CUDA graph per token slot: the forward as a deployment would replay it
    graphs = []
    for j in range(n_pool):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(j)
        graphs.append(g)
    n_prof = min(n_pool, 16)
    prof_graphs, prof_ev = [], []
    if wl.layers == 1:
        for j in range(n_prof):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(cm.COLI_STAGES + 1)]
            for e in ev:
                e.record(stream)          # create the CUDA events outside the capture
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(j, ev)
            prof_graphs.append(g)
            prof_ev.append(ev)
    for j in range(n_pool):
        graphs[j].replay()
    torch.cuda.synchronize()

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush.zero_()
            starts[i].record(stream)
            graphs[i % n_pool].replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    job_ms = max_over_ranks(total_ms, world, dev)
    # the median step of the slowest rank
    job_med = max_over_ranks(statistics.median(step_ms), world, dev)
    value = job_tokens_per_s(T, world, job_med)

    # per-stage device times: graphs with event nodes at the stage boundaries
    st_ms = []
    for i in range(max(n_prof, min(K, 4 * n_prof)) if prof_graphs else 0):
        j = i % n_prof
        flush.zero_()
        prof_graphs[j].replay()
        torch.cuda.synchronize()
        st_ms.append([prof_ev[j][s].elapsed_time(prof_ev[j][s + 1])
                      for s in range(cm.COLI_STAGES)] + [j])
    st_ms = np.array(st_ms)

    # end to end through the host-buffer entry points: each step copies its
    # tokens from pinned host memory into the workspace, runs the layer(s) and
    # copies y back to pinned host memory; the call is captured once per token
    # slot and replayed, as a serving loop would
    xh = torch.empty((n_pool, T, wl.H), dtype=xpool.dtype, pin_memory=True)
    xh.copy_(xpool.cpu())
    yh = torch.empty((T, wl.H), dtype=torch.float32, pin_memory=True)

    def host_step(j):
        if wl.layers == 1:
            cm.coli_moe_forward_host(L0.handle, xh[j], T, yh, ws, path=path)
        else:
            cm.coli_moe_stack_forward_host(handles, xh[j], yh, T, wl.eps, ws, path=path)

    for j in range(min(n_pool, 3)):
        host_step(j)
    torch.cuda.synchronize()
    e2e_graphs = []
    for j in range(n_pool):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            host_step(j)
        e2e_graphs.append(g)
    for j in range(n_pool):
        e2e_graphs[j].replay()
    torch.cuda.synchronize()
    e2e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e2e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        e2e_s[i].record(stream)
        e2e_graphs[i % n_pool].replay()
        e2e_e[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_med = statistics.median(s.elapsed_time(e) for s, e in zip(e2e_s, e2e_e))
    e2e_value = job_tokens_per_s(T, world, max_over_ranks(e2e_med, world, dev))
    # the same steps on the host's clock: each replay is submitted and waited
    # for (after the flush has finished), so host submission counts too
    wall = []
    barrier()
    for i in range(K):
        flush.zero_()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e2e_graphs[i % n_pool].replay()
        torch.cuda.synchronize()
        wall.append((time.perf_counter() - t0) * 1e3)
    barrier()
    wall_ms = max_over_ranks(statistics.median(wall), world, dev)
    e2e_wall = {"value": job_tokens_per_s(T, world, wall_ms), "unit": UNIT, "ms_per_step": wall_ms,
                "timing": "host perf_counter around each replay and its synchronize, median"}

    # bytes: int4 codes + f32 scales of the unique routed experts + shared, per step
    blob = L0.blob_bytes
    hbm_gbs, bf16_tf, peak_src = measured_peaks()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": job_med, "mean_ms_per_step": job_ms / K,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded SplitMix64/Box-Muller, random-init weights)"}
    cfg = {"workload": wl.name, "tokens_per_step": T, "hidden": wl.H, "experts": wl.E,
           "top_k": wl.k, "intermediate": wl.I, "shared": wl.n_shared,
           "scale_group": wl.group or "per-row", "layers": wl.layers,
           "x_dtype": wl.x_dtype, "path": args.path, "path_taken": resolved,
           "weight_bits": args.bits,
           "topp": args.topp or None,
           "l2": "256 MiB buffer written between timed steps (flush), not timed",
           "launch": "one CUDA graph per token slot, replayed",
           "e2e_launch": ("coli_moe_forward_host / coli_moe_stack_forward_host (pinned host x "
                          "and y), captured as one CUDA graph per token slot, replayed")}
    if wl.layers == 1:
        uniq_slot = np.array([len(np.unique(slot_idx[j][slot_w[j] != 0])) for j in range(n_pool)])
        uniq = uniq_slot[np.arange(K) % n_pool]
        nbytes = (uniq + wl.n_shared) * blob
        weight_gbs = nbytes.sum() / (total_ms / 1e3) / 1e9
        ng_h = 1 if wl.group == 0 else wl.H // wl.group
        ng_i = 1 if wl.group == 0 else wl.I // wl.group
        gu_bytes_unit = 2 * (wl.I * wl.H * args.bits // 8 + wl.I * ng_h * 4)
        dn_bytes_unit = wl.H * wl.I * args.bits // 8 + wl.H * ng_i * 4
        units = uniq_slot[st_ms[:, -1].astype(int)] + wl.n_shared
        stage_mean = st_ms[:, :-1].mean(0)
        if fused:
            # moe_fused_kernel (top-k, union, gate/up, down partials) is the
            # "gateup" stage, moe_combine_kernel the "combine" stage
            kern_bytes = units * (gu_bytes_unit + dn_bytes_unit)
            ach = kern_bytes.sum() / (st_ms[:, 2].sum() / 1e3) / 1e9
            kname = "moe_fused_kernel (top-k, union, gate/up, down partial products)"
            line["stages_us"] = {"router": 1e3 * stage_mean[0], "fused": 1e3 * stage_mean[2],
                                 "combine": 1e3 * stage_mean[4]}
        else:
            gu_ach = (units * gu_bytes_unit).sum() / (st_ms[:, 2].sum() / 1e3) / 1e9
            dn_ach = (units * dn_bytes_unit).sum() / (st_ms[:, 3].sum() / 1e3) / 1e9
            dominant = "gateup" if stage_mean[2] >= stage_mean[3] else "down"
            ach = gu_ach if dominant == "gateup" else dn_ach
            kern_bytes = units * (gu_bytes_unit if dominant == "gateup" else dn_bytes_unit)
            gemm = resolved == "gemm"
            two = resolved == "twopass"
            part = "gate/up" if dominant == "gateup" else "down"
            kname = (f"moe_gemm_kernel ({part})" if gemm else
                     (f"moe_split_kernel ({part} pass)" if two else f"{dominant}_gemv_kernel"))
            line["stages_us"] = {n: 1e3 * v for n, v in zip(cm.STAGE_NAMES, stage_mean)}
            line["down_gbs"] = dn_ach
            if gemm or two:
                # tensor work of the dominant launch: gate/up is 2I x H per pair, down H x I
                pairs = T * (wl.k + wl.n_shared)
                rows_k = 2 * wl.I * wl.H if dominant == "gateup" else wl.H * wl.I
                col = 2 if dominant == "gateup" else 3
                tflops = 2.0 * pairs * rows_k / (st_ms[:, col].mean() / 1e3) / 1e12
                if gemm:
                    line["tensor_roofline"] = {"bound": "tensor", "achieved": tflops,
                                               "peak": bf16_tf, "unit": "TFLOP/s",
                                               "frac": tflops / bf16_tf, "kernel": kname,
                                               "dtype": "f16 x f16 -> f32", "peak_source": peak_src}
                else:
                    # mma.sync s8 with two activation digits: two s8 products per
                    # product of the layer; peak: the measured bf16 peak x 2
                    # (the nominal dense int8 : bf16 ratio)
                    line["tensor_roofline"] = {"bound": "tensor", "achieved": tflops,
                                               "peak": 2 * bf16_tf, "unit": "TOP/s",
                                               "frac": tflops / (2 * bf16_tf), "kernel": kname,
                                               "dtype": "s8 x s8 -> s32 (two activation digits)",
                                               "peak_source": peak_src + " bf16 x 2"}
        traffic = None
        if fused and wl.name == "glm_decode" and T == 1 and not args.topp:
            traffic = profiled_traffic("int4_routed_expert_top_b200/csrc/fused.cuh",
                                       "moe_fused_kernel_glm_decode_int8.md" if args.bits == 8
                                       else "moe_fused_kernel_glm_decode.md")
        line["roofline"] = {"bound": "hbm", "achieved": ach, "peak": hbm_gbs, "unit": "GB/s",
                            "frac": ach / hbm_gbs, "traffic": traffic, "kernel": kname,
                            "peak_source": peak_src,
                            "frac_of_spec": ach / SPEC_HBM_GBS,
                            "traffic_source": ("ncu summary in profiles/ for this kernel "
                                               "source (hash-matched)" if traffic else None),
                            "bytes_per_launch": float(kern_bytes.mean())}
        line["int4_weight_gbs"] = weight_gbs
        line["int4_weight_frac_of_hbm"] = weight_gbs / hbm_gbs
        line["int4_weight_frac_of_spec"] = weight_gbs / SPEC_HBM_GBS
        line["unique_experts_per_step"] = float(uniq.mean())
        line["gpu_launches"] = launches_per_layer(wl, T, args.path, fused) * K
    else:   # per layer: the RMSNorm, then the path's own launches
        line["gpu_launches"] = (1 + launches_per_layer(wl, T, args.path, fused)) * wl.layers * K
    line["config"] = cfg
    line["clocks"] = clocks.summary()
    line["e2e"] = {"value": e2e_value, "unit": UNIT,
                   "h2d_bytes_per_step": int(xpool[0].numel() * xpool.element_size()),
                   "d2h_bytes_per_step": int(T * wl.H * 4),
                   "wall_clock": e2e_wall}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, n, secs, smp = oracle_sample(wl)
        threads = oracle_threads()
        par_rate, par_n, par_s = oracle_sample_parallel(smp, threads)
        stack = (f"; one layer per token, the rate divided by the {wl.layers} layers of the "
                 f"stack (every layer has the same shapes)" if wl.layers > 1 else "")
        line["cpu_baseline"] = {
            "value": par_rate / wl.layers, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{par_n} tokens of {wl.name} through the oracle on {threads} host threads "
                      f"at once ({par_s:.1f} s wall), parallel over tokens: router over all "
                      f"{wl.E} experts, dequantisation of the {wl.k}+{wl.n_shared} experts each "
                      f"token uses, SwiGLU, combine{stack}",
            "single_thread": {"value": tok_s / wl.layers, "unit": UNIT, "cores": 1,
                              "sample": f"{n} tokens, {secs:.1f} s"},
            "host": host_cpu()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for l in layers:
        l.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
