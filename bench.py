#!/usr/bin/env python
"""Benchmark of the routed int4 MoE layer (libcolimoe) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--tokens T] [--path auto|gemv|gemm] [--impl own|reference]

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


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
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


def build_layers(wl, device):
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
            routed_scale=wl.routed_scale, norm_topk=wl.norm_topk, device=device))
    return layers


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------
def oracle_sample(wl, T, budget_s=12.0, max_tokens=None):
    """Time the oracle on whole tokens of the workload until ~budget_s of CPU
    work: routing on the full router, dequantisation of every expert matrix the
    token uses, the SwiGLU experts and the combine.  Returns (tokens/s, n, secs)."""
    import oracle
    import synth
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wr, b = synth.router(wl, 0)
    wr_np, b_np = wr.numpy(), b.numpy()
    x = synth.tokens(wl, max(T, 1), layer=0, step=0).numpy()
    cont = {}

    def container(e):   # untimed: the container is built offline
        if e not in cont:
            cont[e] = []
            for t in (synth.T_GATE, synth.T_UP, synth.T_DOWN):
                m = synth.expert_master(wl, 0, t, e, device=dev).cpu().numpy()
                cont[e].append((oracle.quantize(m, wl.group), m.shape[1]))
        return cont[e]

    done, spent = 0, 0.0
    limit = max_tokens or x.shape[0]
    while done < limit and (spent < budget_s or done == 0):
        t = done % x.shape[0]
        idx, w, _ = oracle.route(x[t:t + 1], wr_np, b_np, wl.k)
        experts_ids = [int(e) for e in idx[0]] + [wl.E + s for s in range(wl.n_shared)]
        for e in experts_ids:
            container(e)
        t0 = time.perf_counter()
        idx, w, _ = oracle.route(x[t:t + 1], wr_np, b_np, wl.k)
        ex = []
        for e in experts_ids:
            ex.append(tuple(oracle.dequantize(p, s, K, wl.group) for (p, s), K in container(e)))
        oracle.token_forward(x[t], w[0], ex, wl.n_shared)
        spent += time.perf_counter() - t0
        done += 1
    return done / spent, done, spent


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(args.workload)
    T = args.tokens or wl.T
    per_step = []
    n_steps = args.warmup + args.steps
    t_all = time.perf_counter()
    for i in range(n_steps):
        if time.perf_counter() - t_all > 150 and i >= args.warmup + 1:
            break                       # keep the reference arm within a few minutes
        _, n, secs = oracle_sample(wl, T, budget_s=0.0, max_tokens=1)
        if i >= args.warmup:
            per_step.append(secs)
    tok_s = len(per_step) / sum(per_step)
    sample = (f"{len(per_step)} timed steps of 1 token each (router over all {wl.E} experts, "
              f"dequantisation of the {wl.k}+{wl.n_shared} expert matrices it uses, SwiGLU, "
              f"combine) of workload {wl.name}")
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT,
            "n_gpus": args.gpus, "steps": len(per_step), "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(per_step) / len(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens_per_step": 1},
            "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# own arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="glm_decode")
    ap.add_argument("--tokens", type=int, default=0, help="override tokens per step")
    ap.add_argument("--path", default="auto", choices=("auto", "gemv", "gemm"))
    ap.add_argument("--impl", default="own", choices=("own", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)

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
    T = args.tokens or wl.T
    path = {"auto": cm.COLI_PATH_AUTO, "gemv": cm.COLI_PATH_GEMV, "gemm": cm.COLI_PATH_GEMM}[args.path]
    layers = build_layers(wl, dev)
    L0 = layers[0]
    n_pool = 64 if T <= 16 else 2
    xpool = token_pool(wl, T, n_pool, rank, dev)
    y = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    xs = torch.empty((T, wl.H), dtype=torch.float32, device=dev)   # stack residual stream
    ws = torch.empty((max(cm.coli_moe_stack_workspace_size([l.handle for l in layers], T)
                          if wl.layers > 1 else 0, L0.workspace_bytes(T)),),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    idx_all = torch.empty((args.steps, T, wl.k), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, events=None, record_idx=False):
        xi = xpool[i % n_pool]
        if wl.layers == 1:
            cm.coli_moe_forward_ex(L0.handle, xi, T, y, ws, path=path,
                                   idx_out=idx_all[i] if record_idx else None, events=events)
        else:
            xs.copy_(xi)
            cm.coli_moe_stack_forward([l.handle for l in layers], xs, T, wl.eps, ws, path=path)

    for i in range(args.warmup):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stage_ev = ([[torch.cuda.Event(enable_timing=True) for _ in range(cm.COLI_STAGES + 1)]
                 for _ in range(K)] if wl.layers == 1 else None)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush.zero_()
            starts[i].record(stream)
            step(i, stage_ev[i] if stage_ev else None, record_idx=wl.layers == 1)
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    tot = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tot, op=dist.ReduceOp.MAX)
    job_ms = float(tot.item())
    tokens_all = T * K * world
    value = tokens_all / (job_ms / 1e3)

    # end to end through the public API: pinned host x -> device, forward, y -> host
    xh = torch.empty((n_pool, T, wl.H), dtype=xpool.dtype, pin_memory=True)
    xh.copy_(xpool.cpu())
    yh = torch.empty((T, wl.H), dtype=torch.float32, pin_memory=True)
    xd = torch.empty_like(xpool[0])
    e2e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e2e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        e2e_s[i].record(stream)
        xd.copy_(xh[i % n_pool], non_blocking=True)
        if wl.layers == 1:
            cm.coli_moe_forward_ex(L0.handle, xd, T, y, ws, path=path)
        else:
            xs.copy_(xd)
            cm.coli_moe_stack_forward([l.handle for l in layers], xs, T, wl.eps, ws, path=path)
        yh.copy_(y if wl.layers == 1 else xs, non_blocking=True)
        e2e_e[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = sum(s.elapsed_time(e) for s, e in zip(e2e_s, e2e_e))
    t2 = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t2, op=dist.ReduceOp.MAX)
    e2e_value = tokens_all / (float(t2.item()) / 1e3)

    # bytes: int4 codes + f32 scales of the unique routed experts + shared, per step
    blob = L0.blob_bytes
    hbm_gbs, bf16_tf, peak_src = measured_peaks()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": job_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded SplitMix64/Box-Muller, random-init weights)"}
    cfg = {"workload": wl.name, "tokens_per_step": T, "hidden": wl.H, "experts": wl.E,
           "top_k": wl.k, "intermediate": wl.I, "shared": wl.n_shared,
           "scale_group": wl.group or "per-row", "layers": wl.layers,
           "x_dtype": wl.x_dtype, "path": args.path,
           "l2": "256 MiB buffer written between timed steps (flush), not timed"}
    if wl.layers == 1:
        idx_np = idx_all.cpu().numpy()
        uniq = np.array([len(np.unique(idx_np[i])) for i in range(K)])
        nbytes = (uniq + wl.n_shared) * blob
        weight_gbs = nbytes.sum() / (total_ms / 1e3) / 1e9
        st_ms = np.array([[stage_ev[i][s].elapsed_time(stage_ev[i][s + 1])
                           for s in range(cm.COLI_STAGES)] for i in range(K)])
        stage_mean = st_ms.mean(0)
        L = L0.desc
        gu_bytes_unit = 2 * (wl.I * wl.H // 2 + wl.I * (1 if wl.group == 0 else wl.H // wl.group) * 4)
        dn_bytes_unit = wl.H * wl.I // 2 + wl.H * (1 if wl.group == 0 else wl.I // wl.group) * 4
        units = uniq + wl.n_shared
        gu_ach = (units * gu_bytes_unit / (st_ms[:, 2] / 1e3)).mean() / 1e9
        dn_ach = (units * dn_bytes_unit / (st_ms[:, 3] / 1e3)).mean() / 1e9
        dominant = "gateup" if stage_mean[2] >= stage_mean[3] else "down"
        ach = gu_ach if dominant == "gateup" else dn_ach
        line["roofline"] = {"bound": "hbm", "achieved": ach, "peak": hbm_gbs, "unit": "GB/s",
                            "frac": ach / hbm_gbs, "traffic": None,
                            "kernel": f"expert_gemv_kernel ({dominant})",
                            "peak_source": peak_src}
        line["stages_us"] = {n: 1e3 * v for n, v in zip(cm.STAGE_NAMES, stage_mean)}
        line["int4_weight_gbs"] = weight_gbs
        line["int4_weight_frac_of_hbm"] = weight_gbs / hbm_gbs
        line["unique_experts_per_step"] = float(uniq.mean())
        line["gpu_launches"] = 6 * K
    else:
        line["gpu_launches"] = 7 * wl.layers * K
    line["config"] = cfg
    line["clocks"] = clocks.summary()
    line["e2e"] = {"value": e2e_value, "unit": UNIT,
                   "h2d_bytes_per_step": int(xpool[0].numel() * xpool.element_size()),
                   "d2h_bytes_per_step": int(T * wl.H * 4)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, n, secs = oracle_sample(wl, T)
        line["cpu_baseline"] = {
            "value": tok_s, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of {wl.name} through the oracle ({secs:.1f} s): router over "
                      f"all {wl.E} experts, dequantisation of the {wl.k}+{wl.n_shared} experts "
                      f"each token uses, SwiGLU, combine; single-threaded (one token)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for l in layers:
        l.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
