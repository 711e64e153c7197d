"""Python handle on the plain-C oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product library
never does, and it shares no code with it.  Arguments are numpy arrays; every
function returns fresh arrays and raises on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2 -fopenmp -ffp-contract=off)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.orc_quantize.argtypes = [P, i64, i64, ctypes.c_int32, P, P]
        L.orc_dequantize.argtypes = [P, P, i64, i64, ctypes.c_int32, P]
        L.orc_route.argtypes = [P, i64, i64, P, P, i64, i64, ctypes.c_double,
                                ctypes.c_int, P, P, P]
        L.orc_union.argtypes = [P, i64, i64, i64, P, P, P, P, P]
        L.orc_expert.argtypes = [P, i64, i64, P, P, P, P, i64, P]
        L.orc_token_forward.argtypes = [P, i64, i64, i64, P, P, P, P, i64, P, i64, P]
        L.orc_layer_forward.argtypes = [P, i64, i64, i64, i64, i64, i64,
                                        ctypes.c_int32, ctypes.c_double, ctypes.c_int,
                                        P, P, P, P, P, P, P, P]
        L.orc_rmsnorm.argtypes = [P, i64, i64, ctypes.c_double, P]
        L.orc_fp8_block_dequant.argtypes = [P, P, i64, i64, P]
        L.orc_topp_keep.argtypes = [P, P, i64, ctypes.c_double, P]
        L.orc_quantize8.argtypes = [P, i64, i64, ctypes.c_int32, P, P]
        L.orc_dequantize8.argtypes = [P, P, i64, i64, ctypes.c_int32, P]
        L.orc_topp_keep.restype = i64
        for f in ("orc_quantize", "orc_dequantize", "orc_route", "orc_union",
                  "orc_expert", "orc_token_forward", "orc_layer_forward",
                  "orc_rmsnorm", "orc_fp8_block_dequant", "orc_quantize8", "orc_dequantize8"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def quantize(w, group: int):
    w, pw = _c(w, np.float32)
    rows, cols = w.shape
    ng = 1 if group == 0 else cols // group
    packed = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, ng), np.float32)
    _check(lib().orc_quantize(pw, rows, cols, group, packed.ctypes.data_as(ctypes.c_void_p),
                              scales.ctypes.data_as(ctypes.c_void_p)), "quantize")
    return packed, scales


def fp8_block_dequant(codes, block_scales):
    """FP8 E4M3 codes [R, K] (uint8) with one f32 scale per 128 x 128 block
    ([ceil(R/128), ceil(K/128)]) -> f32 [R, K]."""
    codes, pq = _c(codes, np.uint8)
    bs, pb = _c(block_scales, np.float32)
    rows, cols = codes.shape
    assert bs.shape == ((rows + 127) // 128, (cols + 127) // 128)
    out = np.zeros((rows, cols), np.float32)
    _check(lib().orc_fp8_block_dequant(pq, pb, rows, cols, out.ctypes.data_as(ctypes.c_void_p)),
           "fp8_block_dequant")
    return out


def quantize8(w, group: int):
    """8-bit container: signed byte codes [R, K] and f32 scales [R, K/G]."""
    w, pw = _c(w, np.float32)
    rows, cols = w.shape
    ng = 1 if group == 0 else cols // group
    codes = np.zeros((rows, cols), np.int8)
    scales = np.zeros((rows, ng), np.float32)
    _check(lib().orc_quantize8(pw, rows, cols, group, codes.ctypes.data_as(ctypes.c_void_p),
                               scales.ctypes.data_as(ctypes.c_void_p)), "quantize8")
    return codes, scales


def dequantize8(codes, scales, group: int):
    codes, pc = _c(codes, np.int8)
    scales, ps = _c(scales, np.float32)
    rows, cols = codes.shape
    out = np.zeros((rows, cols), np.float32)
    _check(lib().orc_dequantize8(pc, ps, rows, cols, group, out.ctypes.data_as(ctypes.c_void_p)),
           "dequantize8")
    return out


def topp_keep(w, idx, p: float):
    """Adaptive expert top-p: w, idx [T, k] (routing weights, experts, pick
    order) -> keep [T, k] int32 (1 kept) and the number kept per token."""
    w, pw = _c(np.atleast_2d(w), np.float32)
    idx, pi = _c(np.atleast_2d(idx), np.int32)
    T, k = w.shape
    keep = np.zeros((T, k), np.int32)
    n = np.zeros(T, np.int64)
    for t in range(T):
        r = lib().orc_topp_keep(w[t].ctypes.data_as(ctypes.c_void_p),
                                idx[t].ctypes.data_as(ctypes.c_void_p), k, float(p),
                                keep[t].ctypes.data_as(ctypes.c_void_p))
        _check(0 if r >= 1 else -1, "topp_keep")
        n[t] = r
    return keep, n


def dequantize(packed, scales, cols: int, group: int):
    packed, pp = _c(packed, np.uint8)
    scales, ps = _c(scales, np.float32)
    rows = packed.shape[0]
    out = np.zeros((rows, cols), np.float32)
    _check(lib().orc_dequantize(pp, ps, rows, cols, group,
                                out.ctypes.data_as(ctypes.c_void_p)), "dequantize")
    return out


def route(x, wr, bias, k: int, routed_scale: float = 1.0, norm_topk: bool = True):
    x, px = _c(x, np.float32)
    wr, pwr = _c(wr, np.float32)
    bias, pb = _c(bias, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    gap = np.zeros((T,), np.float64)
    _check(lib().orc_route(px, T, H, pwr, pb, E, k, routed_scale, int(norm_topk),
                           idx.ctypes.data_as(ctypes.c_void_p),
                           w.ctypes.data_as(ctypes.c_void_p),
                           gap.ctypes.data_as(ctypes.c_void_p)), "route")
    return idx, w, gap


def union(idx, E: int):
    idx, pi = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.zeros((E + 1,), np.int32)
    pair_tok = np.zeros((max(T * k, 1),), np.int32)
    pair_slot = np.zeros((max(T * k, 1),), np.int32)
    uniq = np.zeros((E,), np.int32)
    n_uniq = np.zeros((1,), np.int32)
    _check(lib().orc_union(pi, T, k, E, *(a.ctypes.data_as(ctypes.c_void_p) for a in
                                          (offsets, pair_tok, pair_slot, uniq, n_uniq))),
           "union")
    n = int(n_uniq[0])
    return offsets, pair_tok[: T * k], pair_slot[: T * k], uniq[:n], n


def expert(x, wg, wu, wd, rows=None):
    x, px = _c(x, np.float32)
    wg, pg = _c(wg, np.float32)
    wu, pu = _c(wu, np.float32)
    wd, pd = _c(wd, np.float32)
    I, H = wg.shape
    if rows is None:
        prow, n = None, H
    else:
        rows, prow = _c(rows, np.int32)
        n = rows.shape[0]
    o = np.zeros((n,), np.float64)
    _check(lib().orc_expert(px, H, I, pg, pu, pd, prow, n,
                            o.ctypes.data_as(ctypes.c_void_p)), "expert")
    return o


def token_forward(x, w, experts, n_shared: int, rows=None):
    """experts: list of (gate, up, down) dequantised f32 matrices, the k routed
    experts of this token in slot order followed by the shared experts."""
    x, px = _c(x, np.float32)
    w, pw = _c(w, np.float32)
    k = w.shape[0]
    assert len(experts) == k + n_shared
    keep = [tuple(np.ascontiguousarray(m, np.float32) for m in e) for e in experts]
    I, H = keep[0][0].shape
    arr = ctypes.c_void_p * len(keep)
    pg = arr(*[e[0].ctypes.data for e in keep])
    pu = arr(*[e[1].ctypes.data for e in keep])
    pd = arr(*[e[2].ctypes.data for e in keep])
    if rows is None:
        prow, n = None, H
    else:
        rows, prow = _c(rows, np.int32)
        n = rows.shape[0]
    y = np.zeros((n,), np.float32)
    _check(lib().orc_token_forward(px, H, I, k, pw, pg, pu, pd, n_shared, prow, n,
                                   y.ctypes.data_as(ctypes.c_void_p)), "token_forward")
    return y


def layer_forward(x, wr, bias, gate_m, up_m, down_m, k: int, n_shared: int, group: int,
                  routed_scale: float = 1.0, norm_topk: bool = True):
    x, px = _c(x, np.float32)
    wr, pwr = _c(wr, np.float32)
    bias, pb = _c(bias, np.float32)
    gate_m, pg = _c(gate_m, np.float32)
    up_m, pu = _c(up_m, np.float32)
    down_m, pd = _c(down_m, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    I = gate_m.shape[1]
    assert gate_m.shape == (E + n_shared, I, H) and down_m.shape == (E + n_shared, H, I)
    y = np.zeros((T, H), np.float32)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    _check(lib().orc_layer_forward(px, T, H, I, E, k, n_shared, group, routed_scale,
                                   int(norm_topk), pwr, pb, pg, pu, pd,
                                   y.ctypes.data_as(ctypes.c_void_p),
                                   idx.ctypes.data_as(ctypes.c_void_p),
                                   w.ctypes.data_as(ctypes.c_void_p)), "layer_forward")
    return y, idx, w


def rmsnorm(x, eps: float = 1e-5):
    x, px = _c(x, np.float32)
    T, H = x.shape
    out = np.zeros_like(x)
    _check(lib().orc_rmsnorm(px, T, H, eps, out.ctypes.data_as(ctypes.c_void_p)), "rmsnorm")
    return out
