"""Seeded synthetic inputs for the routed int4 MoE layer.

This module only draws random numbers and names the workloads; it holds none
of the method's arithmetic (no quantisation, routing or expert math), so both
the CUDA path and the CPU oracle may take their inputs from it.

Generator: counter-based SplitMix64.  A stream is keyed by
(seed, layer, tensor, expert, row); its i-th 64-bit draw is
mix(key + (i + 1) * GOLDEN).  Uniforms are the top 53 bits scaled by 2**-53;
normals use Box-Muller in double on draws (2i, 2i+1):
sqrt(-2 ln(1 - u0)) * cos(2 pi u1), then cast to f32 by the caller.
Draws are made with torch int64 ops (wrapping two's complement), so the same
code runs on the CPU or on a CUDA device; a given test always hands the very
same generated tensor to both sides.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field

import torch

GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_U64 = 1 << 64

# tensor ids of the streams
T_ROUTER, T_BIAS, T_GATE, T_UP, T_DOWN, T_X, T_PERM = 1, 2, 3, 4, 5, 6, 7


def _s64(v: int) -> int:
    v %= _U64
    return v - _U64 if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z: torch.Tensor) -> torch.Tensor:
    z = z ^ _lsr(z, 30)
    z = z * _s64(_M1)
    z = z ^ _lsr(z, 27)
    z = z * _s64(_M2)
    return z ^ _lsr(z, 31)


def mix_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (reference for the tensor version)."""
    z %= _U64
    z = ((z ^ (z >> 30)) * _M1) % _U64
    z = ((z ^ (z >> 27)) * _M2) % _U64
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int, tensor: int, expert: int, row: int) -> int:
    key = seed % _U64
    for f in (layer, tensor, expert, row):
        key = mix_int(key + (f + 1) * GOLDEN)
    return key


def _keys(seed, layer, tensor, expert, rows: torch.Tensor) -> torch.Tensor:
    base = seed % _U64
    for f in (layer, tensor, expert):
        base = mix_int(base + (f + 1) * GOLDEN)
    return _mix_t(torch.full_like(rows, _s64(base)) + (rows + 1) * _s64(GOLDEN))


def _draws(keys: torch.Tensor, first: int, n: int) -> torch.Tensor:
    i = torch.arange(first + 1, first + n + 1, device=keys.device, dtype=torch.int64)
    return _mix_t(keys[:, None] + i[None, :] * _s64(GOLDEN))


def _unit(bits: torch.Tensor) -> torch.Tensor:
    return _lsr(bits, 11).to(torch.float64) * (2.0 ** -53)


def uniform(seed, layer, tensor, expert, rows, cols, device="cpu", first=0):
    """[len(rows), cols] float64 uniforms in [0, 1)."""
    rows = torch.as_tensor(rows, dtype=torch.int64, device=device).reshape(-1)
    return _unit(_draws(_keys(seed, layer, tensor, expert, rows), first, cols))


def normal(seed, layer, tensor, expert, rows, cols, device="cpu", first=0):
    """[len(rows), cols] float64 standard normals (Box-Muller, cosine branch).
    ``first`` counts normals already consumed from each row's stream."""
    rows = torch.as_tensor(rows, dtype=torch.int64, device=device).reshape(-1)
    u = _unit(_draws(_keys(seed, layer, tensor, expert, rows), 2 * first, 2 * cols))
    u0, u1 = u[:, 0::2], u[:, 1::2]
    return torch.sqrt(-2.0 * torch.log1p(-u0)) * torch.cos((2.0 * math.pi) * u1)


# ---------------------------------------------------------------------------
# Workloads (the layer shapes and input recipes of the GLM-5.2-shaped layer)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    k: int
    n_shared: int
    group: int              # 0 = per-row scale, 64 = one scale per 64 columns
    T: int                  # tokens per forward call
    steps: int = 1          # independent token batches (MTP verify: 64)
    layers: int = 1
    x_dtype: str = "f32"    # "f32" or "bf16"
    bias: str = "uniform"   # "uniform" U(-0.01, 0.01) or "zipf"
    seed: int = 0
    w_std: float = 0.02
    routed_scale: float = 1.0
    norm_topk: bool = True
    eps: float = 1e-5
    sweep: tuple = field(default_factory=tuple)

    @property
    def n_exp(self) -> int:
        return self.E + self.n_shared


TINY = Workload("tiny", H=256, I=128, E=16, k=4, n_shared=1, group=0, T=4, seed=1001)
GLM_DECODE = Workload("glm_decode", H=6144, I=2048, E=256, k=8, n_shared=1, group=0,
                      T=1, seed=2002)
GLM_MTP = Workload("glm_mtp_verify", H=6144, I=2048, E=256, k=8, n_shared=1, group=64,
                   T=3, steps=64, seed=3003)
GLM_PREFILL = Workload("glm_prefill", H=6144, I=2048, E=256, k=8, n_shared=1, group=64,
                       T=512, x_dtype="bf16", bias="zipf", seed=4004)
GLM_STACK = Workload("glm_stack16", H=6144, I=2048, E=256, k=8, n_shared=1, group=64,
                     T=1, layers=16, seed=5005, sweep=(1, 4, 16, 64, 512))

WORKLOADS = {w.name: w for w in (TINY, GLM_DECODE, GLM_MTP, GLM_PREFILL, GLM_STACK)}

_ZIPF_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json")


def zipf_beta(wl: Workload) -> float:
    """Bias amplitude of the Zipf-skewed router (written by oracle/fit_zipf_beta.py)."""
    with open(_ZIPF_FILE) as f:
        return float(json.load(f)[wl.name]["beta"])


def expert_master(wl: Workload, layer: int, tensor: int, expert: int, rows=None,
                  device="cpu") -> torch.Tensor:
    """f32 master weights N(0, w_std) of one expert matrix (all rows, or a subset)."""
    R, C = (wl.I, wl.H) if tensor in (T_GATE, T_UP) else (wl.H, wl.I)
    if rows is None:
        rows = torch.arange(R, device=device)
    return (wl.w_std * normal(wl.seed, layer, tensor, expert, rows, C, device)).to(torch.float32)


def router(wl: Workload, layer: int = 0, device="cpu", beta: float | None = None):
    """Router weights W_r [E, H] f32 N(0, w_std) and selection bias [E] f32."""
    wr = (wl.w_std * normal(wl.seed, layer, T_ROUTER, 0, torch.arange(wl.E, device=device),
                            wl.H, device)).to(torch.float32)
    if wl.bias == "zipf":
        keys = uniform(wl.seed, layer, T_PERM, 0, [0], wl.E, device)[0]
        order = torch.argsort(keys, stable=True)
        rank = torch.empty(wl.E, dtype=torch.float64, device=device)
        rank[order] = torch.arange(1, wl.E + 1, dtype=torch.float64, device=device)
        b = (zipf_beta(wl) if beta is None else beta) * rank.pow(-1.1)
    else:
        b = -0.01 + 0.02 * uniform(wl.seed, layer, T_BIAS, 0, [0], wl.E, device)[0]
    return wr, b.to(torch.float32)


def tokens(wl: Workload, T: int, layer: int = 0, step: int = 0, redraw=None,
           device="cpu") -> torch.Tensor:
    """x [T, H] N(0, 1) as f32 (or bf16-rounded f32 when x_dtype == 'bf16').
    redraw[t] = r takes token t's r-th fresh block of H normals from its stream."""
    rows = torch.arange(step * T, step * T + T, device=device)
    if redraw is None or not any(int(r) for r in redraw):
        x = normal(wl.seed, layer, T_X, 0, rows, wl.H, device)
    else:
        x = torch.stack([normal(wl.seed, layer, T_X, 0, rows[t:t + 1], wl.H, device,
                                first=int(redraw[t]) * wl.H)[0] for t in range(T)])
    x = x.to(torch.float32)
    if wl.x_dtype == "bf16":
        x = x.to(torch.bfloat16).to(torch.float32)
    return x
