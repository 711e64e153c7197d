"""The union a forward builds inside its own workspace, read back after the call
(coli_moe_union_readback), against the oracle's union of the same picks.

The standalone union entry point is tested elsewhere on given picks; this file
checks the one the layer itself uses: on the GEMV and tensor-core paths the
expert offsets, the (token, slot) pairs grouped by expert and the unique-expert
list equal the oracle's stable grouping of the picks the call computes (all
picks, or those top-p or an expert range keep), and every pick's pair index
names its own (token, slot).  The fused path keeps its union in shared memory
and publishes each pick's pair index: with more than 32 picks its grouping is
the same (experts ascending), with at most 32 the experts come in the order
the picks first name them (token, then slot); both are rebuilt here from their
definitions and compared index for index."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
import int4_routed_expert_top_b200 as cm
from int4_routed_expert_top_b200.device_layer import DeviceLayer
from tests.workloads import build_layer, gap_resampled_tokens, masters

pytestmark = pytest.mark.gpu


def forward(L, x, T, path):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, L.k), dtype=torch.float32, device="cuda")
    ws = L.workspace(T)
    cm.coli_moe_forward_ex(L.handle, x, T, y, ws, path=path, idx_out=idx, w_out=w)
    E, Tk = L.E, T * L.k
    out = {n: torch.full((s,), -7, dtype=torch.int32, device="cuda") for n, s in
           (("offsets", E + 1), ("pair_tok", Tk), ("pair_slot", Tk), ("uniq", E),
            ("n_uniq", 1), ("inv", Tk))}
    cm.coli_moe_union_readback(L.handle, T, ws, **out)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), {n: v.cpu().numpy() for n, v in out.items()}


def kept_union(idx, w, E):
    """Oracle union of the computed picks: the picks of weight 0 are given an
    expert id past E, so that the oracle's grouping puts them last, then cut."""
    T, k = idx.shape
    moved = np.where(w != 0, idx, E).astype(np.int32)
    off, ptok, pslot, uniq, n = oracle.union(moved, E + 1)
    used = int(off[E])
    if n and uniq[-1] == E:
        n -= 1
    return off[: E + 1], ptok[:used], pslot[:used], uniq[:n], n


def check_grouped(idx, w, u, E):
    off, ptok, pslot, uniq, n = kept_union(idx, w, E)
    used = int(off[E])
    assert int(u["n_uniq"][0]) == n
    np.testing.assert_array_equal(u["offsets"], off)
    np.testing.assert_array_equal(u["pair_tok"][:used], ptok)
    np.testing.assert_array_equal(u["pair_slot"][:used], pslot)
    np.testing.assert_array_equal(u["uniq"][:n], uniq)
    assert (u["pair_tok"][used:] == 0).all() and (u["pair_slot"][used:] == 0).all()
    check_inv(idx, w, u["inv"])
    inv = u["inv"].reshape(idx.shape)
    t, j = np.nonzero(w != 0)
    np.testing.assert_array_equal(u["pair_tok"][inv[t, j]], t)
    np.testing.assert_array_equal(u["pair_slot"][inv[t, j]], j)


def check_inv(idx, w, inv_flat):
    """Pair indices of the computed picks: 0..n-1 once each, one contiguous run
    per expert with its tokens ascending; -1 for every pick not computed."""
    inv = inv_flat.reshape(idx.shape)
    valid = w != 0
    assert (inv[~valid] == -1).all()
    p = inv[valid]
    np.testing.assert_array_equal(np.sort(p), np.arange(p.size))
    t_of = np.nonzero(valid)[0]
    for e in np.unique(idx[valid]):
        sel = idx[valid] == e
        pe = p[sel]
        order = np.argsort(pe)
        assert pe[order][-1] - pe[order][0] == pe.size - 1, e      # contiguous run
        assert (np.diff(t_of[sel][order]) > 0).all(), e             # tokens ascending


def inv_from_pairs(shape, ptok, pslot):
    inv = np.full(shape, -1, np.int32)
    inv[ptok, pslot] = np.arange(ptok.size, dtype=np.int32)
    return inv


def fused_inv_ref(idx, w, E):
    """Pair index of every pick in the fused kernel's union."""
    T, k = idx.shape
    if T * k > 32:
        _, ptok, pslot, _, _ = kept_union(idx, w, E)
        return inv_from_pairs(idx.shape, ptok, pslot)
    order = []                                   # experts by first naming
    for t in range(T):
        for j in range(k):
            if w[t, j] != 0 and idx[t, j] not in order:
                order.append(int(idx[t, j]))
    ptok, pslot = [], []
    for e in order:
        for t in range(T):
            for j in range(k):
                if w[t, j] != 0 and idx[t, j] == e:
                    ptok.append(t)
                    pslot.append(j)
    return inv_from_pairs(idx.shape, np.array(ptok, np.int64), np.array(pslot, np.int64))


CASES = [dict(T=1), dict(T=5), dict(T=40, group=64), dict(T=60, k=8, E=32, group=64),
         dict(T=150, k=8, E=32, group=64)]


@pytest.mark.parametrize("topp", [0.0, 0.7])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(f"{a}{b}" for a, b in c.items()))
def test_forward_union_matches_oracle(case, topp):
    wl = dataclasses.replace(synth.TINY, **case)
    router = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, wl.T, *router)
    L = build_layer(wl, router=router)
    cm.coli_moe_layer_set_topp(L.handle, topp)
    for path in (cm.COLI_PATH_GEMV, cm.COLI_PATH_GEMM):
        idx, w, u = forward(L, x.cuda(), wl.T, path)
        if topp == 0.0:
            assert (w != 0).all()
            full = oracle.union(idx, wl.E)
            np.testing.assert_array_equal(u["offsets"], full[0])
        check_grouped(idx, w, u, wl.E)
    if wl.T * (wl.k + wl.n_shared) <= 640:                     # the fused path's limit
        idx, w, u = forward(L, x.cuda(), wl.T, cm.COLI_PATH_FUSED)
        check_inv(idx, w, u["inv"])
        np.testing.assert_array_equal(u["inv"].reshape(idx.shape), fused_inv_ref(idx, w, wl.E))
    L.close()


@pytest.mark.parametrize("T", [1, 33])
def test_forward_union_of_an_expert_range(T):
    """A rank holding experts [16, 48) of 64: its union holds only its own picks."""
    wl = dataclasses.replace(synth.TINY, T=T, E=64, k=4, group=64)
    router = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, T, *router)
    L = DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, *router,
                    expert_masters=lambda e: masters(wl, 0, e), expert_range=(16, 48),
                    with_shared=False)
    for path in (cm.COLI_PATH_GEMV, cm.COLI_PATH_GEMM, cm.COLI_PATH_FUSED):
        idx, w, u = forward(L, x.cuda(), T, path)
        inside = (idx >= 16) & (idx < 48)
        np.testing.assert_array_equal(w != 0, inside)
        if path == cm.COLI_PATH_FUSED:
            check_inv(idx, w, u["inv"])
            np.testing.assert_array_equal(u["inv"].reshape(idx.shape),
                                          fused_inv_ref(idx, w, wl.E))
        else:
            check_grouped(idx, w, u, wl.E)
            assert ((u["uniq"][: int(u["n_uniq"][0])] >= 16) &
                    (u["uniq"][: int(u["n_uniq"][0])] < 48)).all()
    L.close()


@pytest.mark.parametrize("topp", [0.0, 0.7])
@pytest.mark.parametrize("T,E,k", [(70, 16, 4), (300, 8, 2)])
def test_two_pass_forward_union_matches_oracle(T, E, k, topp):
    """The two-pass path (I a multiple of 256) builds the same union as the
    GEMV/GEMM paths: units of many 16-pair chunks included."""
    wl = dataclasses.replace(synth.TINY, I=256, T=T, E=E, k=k, group=64)
    router = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, T, *router)
    L = build_layer(wl, router=router)
    cm.coli_moe_layer_set_topp(L.handle, topp)
    idx, w, u = forward(L, x.cuda(), T, cm.COLI_PATH_TWOPASS)
    check_grouped(idx, w, u, wl.E)
    L.close()
