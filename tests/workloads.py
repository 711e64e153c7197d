"""Test harness: seeded layers on the device, oracle references, the gap rule.

Inputs come from ``synth`` only; the device layer is built by the library's own
quantiser; references come from ``oracle`` on the very same master values."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from int4_routed_expert_top_b200.device_layer import DeviceLayer

MATS = (synth.T_GATE, synth.T_UP, synth.T_DOWN)


def rel_err(y, ref) -> float:
    """Norm-wise relative error: max |y - ref| / max |ref|."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-30))


def masters(wl, layer, e, device="cuda"):
    return tuple(synth.expert_master(wl, layer, t, e, device=device) for t in MATS)


def build_layer(wl, layer=0, device="cuda", router=None, masters_device=None, bits=4):
    """Layer on ``device``; its f32 masters are drawn on ``masters_device``
    (default: the same device) and quantised by the library on the device
    (4-bit codes, or 8-bit ones with bits=8)."""
    wr, b = router if router is not None else synth.router(wl, layer)
    md = masters_device or device
    return DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, wr, b,
                       expert_masters=lambda e: tuple(
                           m.to(device) for m in masters(wl, layer, e, md)),
                       routed_scale=wl.routed_scale, norm_topk=wl.norm_topk, device=device,
                       bits=bits)


def gap_resampled_tokens(wl, T, wr, b, layer=0, step=0, max_rounds=64):
    """Draw x; redraw every token whose oracle gap sel_(k) - sel_(k+1) < 1e-3 from
    the next block of its stream.  Returns x (cpu f32), oracle idx, w, redraws."""
    redraw = [0] * T
    wr_np, b_np = wr.cpu().numpy(), b.cpu().numpy()
    for _ in range(max_rounds):
        x = synth.tokens(wl, T, layer, step, redraw)
        idx, w, gap = oracle.route(x.numpy(), wr_np, b_np, wl.k, wl.routed_scale,
                                   wl.norm_topk)
        bad = np.nonzero(gap < 1e-3)[0]
        if bad.size == 0:
            return x, idx, w, redraw
        for t in bad:
            redraw[t] += 1
    raise RuntimeError("gap rule did not converge")


class OracleExperts:
    """Dequantised expert matrices computed by the oracle (the int4 container,
    or the 8-bit one with bits=8), cached per expert."""

    def __init__(self, wl, layer=0, device="cuda", bits=4):
        self.wl, self.layer, self.device, self.bits = wl, layer, device, bits
        self.cache = {}

    def __call__(self, e):
        if e not in self.cache:
            mats = []
            for m in masters(self.wl, self.layer, e, self.device):
                m = m.cpu().numpy()
                if self.bits == 8:
                    q, s = oracle.quantize8(m, self.wl.group)
                    mats.append(oracle.dequantize8(q, s, self.wl.group))
                else:
                    p, s = oracle.quantize(m, self.wl.group)
                    mats.append(oracle.dequantize(p, s, m.shape[1], self.wl.group))
            self.cache[e] = tuple(mats)
        return self.cache[e]


def oracle_tokens(wl, experts: OracleExperts, x, idx, w, rows=None):
    """Oracle outputs [T, n_rows] for tokens x with the oracle's routing."""
    out = []
    shared = [wl.E + s for s in range(wl.n_shared)]
    for t in range(x.shape[0]):
        ex = [experts(int(e)) for e in idx[t]] + [experts(e) for e in shared]
        out.append(oracle.token_forward(x[t], w[t], ex, wl.n_shared, rows))
    return np.stack(out)


def same_selection(idx_gpu, idx_ref, sel_gap_ok=None):
    """Index sets must match exactly; the order must match too (callers pass
    a mask of tokens whose adjacent selected scores differ by >= 1e-6)."""
    a = np.sort(np.asarray(idx_gpu), axis=1)
    b = np.sort(np.asarray(idx_ref), axis=1)
    np.testing.assert_array_equal(a, b)
    if sel_gap_ok is not None:
        np.testing.assert_array_equal(np.asarray(idx_gpu)[sel_gap_ok],
                                      np.asarray(idx_ref)[sel_gap_ok])


def ordered_ok(x, wr, b, idx, k):
    """Tokens whose selected sel values are pairwise >= 1e-6 apart (oracle, double)."""
    z = x.astype(np.float64) @ wr.astype(np.float64).T
    sel = 1 / (1 + np.exp(-z)) + b.astype(np.float64)
    v = np.take_along_axis(sel, idx.astype(np.int64), 1)
    return np.all(np.abs(np.diff(v, axis=1)) >= 1e-6, axis=1)
