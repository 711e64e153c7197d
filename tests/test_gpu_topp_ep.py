"""GPU parity of the picks a call does not compute: adaptive expert top-p
(coli_moe_layer_set_topp) and expert parallelism (coli_moe_layer_set_partition),
on the fused, GEMV and tensor-core paths.

Top-p: the routing itself is unchanged; the kept set of every token equals the
oracle's rule (orc_topp_keep) applied to the very same f32 weights, bit for bit;
kept weights are unchanged; y matches the oracle's forward over the kept
experts only.  Expert parallelism: ranks holding contiguous expert ranges (the
shared experts on rank 0) give partial outputs whose sum is the whole layer's
output, every pick computed by exactly one rank.  The ranks run one after
another on one GPU here; the all-reduce between GPUs is covered by the
world-size-2 gloo test on the CPU."""
import concurrent.futures as cf
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
import int4_routed_expert_top_b200 as cm
from int4_routed_expert_top_b200 import ep
from int4_routed_expert_top_b200.device_layer import DeviceLayer
from tests.workloads import (OracleExperts, build_layer, gap_resampled_tokens, masters,
                             oracle_tokens, rel_err, same_selection)

pytestmark = pytest.mark.gpu

PATHS = {"fused": (cm.COLI_PATH_FUSED, 2e-3), "gemv": (cm.COLI_PATH_GEMV, 2e-3),
         "gemm": (cm.COLI_PATH_GEMM, 1e-2)}


def run(L, x, T, path, residual=None):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, L.k), dtype=torch.float32, device="cuda")
    cm.coli_moe_forward_ex(L.handle, x, T, y, L.workspace(T), residual=residual, path=path,
                           idx_out=idx, w_out=w)
    torch.cuda.synchronize()
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def kept_reference(wl, x, idx_ref, w_ref, idx_gpu, keep_gpu, experts):
    """Oracle forward over the experts the GPU kept (matched by expert id)."""
    w = w_ref.copy()
    for t in range(w.shape[0]):
        kept = set(idx_gpu[t][keep_gpu[t] != 0].tolist())
        for j in range(w.shape[1]):
            if int(idx_ref[t, j]) not in kept:
                w[t, j] = 0.0
    return oracle_tokens(wl, experts, x, idx_ref, w)


def check_topp(wl, L, x, p, paths=PATHS, experts=None):
    T = x.shape[0]
    wr, b = L.router_w.cpu().numpy(), L.router_b.cpu().numpy()
    idx_ref, w_ref, _ = oracle.route(x.numpy(), wr, b, wl.k, wl.routed_scale, wl.norm_topk)
    experts = experts or OracleExperts(wl)
    pf = float(np.float32(p))
    kept_counts = []
    for name, (path, tol) in paths.items():
        cm.coli_moe_layer_set_topp(L.handle, 0.0)
        _, idx_full, w_full = run(L, x.cuda(), T, path)
        cm.coli_moe_layer_set_topp(L.handle, pf)
        y, idx, w = run(L, x.cuda(), T, path)
        cm.coli_moe_layer_set_topp(L.handle, 0.0)
        np.testing.assert_array_equal(idx, idx_full)            # routing unchanged
        same_selection(idx, idx_ref)
        keep, n = oracle.topp_keep(w_full, idx_full, pf)
        np.testing.assert_array_equal((w != 0).astype(np.int32), keep, err_msg=name)
        np.testing.assert_array_equal(w.view(np.uint32)[keep != 0],
                                      w_full.view(np.uint32)[keep != 0])
        y_ref = kept_reference(wl, x.numpy(), idx_ref, w_ref, idx, keep, experts)
        err = rel_err(y, y_ref)
        assert err <= tol, (name, p, err)
        kept_counts.append(n)
    return kept_counts[0]


@pytest.mark.parametrize("p", [0.7, 0.5, 1e-6, 1.0])
@pytest.mark.parametrize("variant", [dict(T=4), dict(T=1, group=64), dict(T=40, group=64),
                                     dict(T=9, k=8, E=32, group=64)])
def test_topp_tiny(variant, p):
    wl = dataclasses.replace(synth.TINY, **variant)
    wr, b = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    L = build_layer(wl, router=(wr, b))
    n = check_topp(wl, L, x, p)
    if p == 1e-6:
        assert (n == 1).all()         # the largest weight alone reaches p
    L.close()


@pytest.fixture(scope="module")
def glm_decode_layer():
    L = build_layer(synth.GLM_DECODE)
    yield L
    L.close()
    torch.cuda.empty_cache()


def test_topp_glm_decode(glm_decode_layer):
    """GLM-5.2 decode layer, p = 0.7: kept sets exact, outputs against the
    oracle's kept-expert forward, and the expert bytes per token against top-8."""
    wl = synth.GLM_DECODE
    L = glm_decode_layer
    experts = OracleExperts(wl)
    total_kept = 0
    steps = 4
    for step in range(steps):
        x, idx_ref, _, _ = gap_resampled_tokens(wl, 1, L.router_w.cpu(), L.router_b.cpu(),
                                                step=step)
        with cf.ThreadPoolExecutor(9) as ex:
            list(ex.map(experts, [int(e) for e in idx_ref[0]] + [wl.E]))
        n = check_topp(wl, L, x, 0.7, paths={"fused": PATHS["fused"], "gemv": PATHS["gemv"]},
                       experts=experts)
        total_kept += int(n[0])
        experts.cache.clear()
    frac = (total_kept / steps + wl.n_shared) / (wl.k + wl.n_shared)
    print(f"top-p 0.7: {total_kept / steps:.2f} routed experts kept per token; expert bytes "
          f"{frac:.3f} of top-8 (shared expert included)")


# ---------------------------------------------------------------------------
# expert parallelism
# ---------------------------------------------------------------------------

def rank_layers(wl, world, router, layer=0):
    wr, b = router
    return [DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, wr, b,
                        expert_masters=lambda e: masters(wl, layer, e),
                        routed_scale=wl.routed_scale, norm_topk=wl.norm_topk,
                        expert_range=ep.expert_range(wl.E, r, world),
                        with_shared=r == ep.SHARED_RANK)
            for r in range(world)]


def check_partition(wl, full, ranks, x, path, tol, residual=None):
    T = x.shape[0]
    y_full, idx_full, w_full = run(full, x, T, path, residual=residual)
    parts, ws = [], []
    for r, L in enumerate(ranks):
        res = residual if r == ep.SHARED_RANK else None
        y, idx, w = run(L, x, T, path, residual=res)
        np.testing.assert_array_equal(idx, idx_full)           # routing is replicated
        lo, hi = L.expert_range
        inside = (idx_full >= lo) & (idx_full < hi)
        np.testing.assert_array_equal(w.view(np.uint32)[inside], w_full.view(np.uint32)[inside])
        assert (w[~inside] == 0).all()
        parts.append(y.astype(np.float64))
        ws.append(w != 0)
    # every computed pick on exactly one rank
    np.testing.assert_array_equal(np.sum(ws, axis=0), (w_full != 0).astype(np.int64))
    total = np.sum(parts, axis=0)
    ref = y_full.astype(np.float64) - (residual.cpu().numpy() if residual is not None else 0)
    err = float(np.abs(total - y_full).max() / np.abs(ref).max())
    assert err <= tol, (path, err)
    return err


@pytest.mark.parametrize("T", [1, 4, 50])
@pytest.mark.parametrize("path", list(PATHS))
def test_expert_parallel_tiny(path, T):
    wl = dataclasses.replace(synth.TINY, group=64, T=T)
    router = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, T, *router)
    full = build_layer(wl, router=router)
    ranks = rank_layers(wl, 4, router)
    res = torch.randn((T, wl.H), device="cuda")
    # the same per-pair products, summed in another order: f32 rounding only
    check_partition(wl, full, ranks, x.cuda(), PATHS[path][0], 2e-5)
    check_partition(wl, full, ranks, x.cuda(), PATHS[path][0], 2e-5, residual=res)
    # top-p decided on the whole routing, then split by expert
    for L in [full] + ranks:
        cm.coli_moe_layer_set_topp(L.handle, 0.7)
    check_partition(wl, full, ranks, x.cuda(), PATHS[path][0], 2e-5)
    for L in [full] + ranks:
        L.close()


def test_expert_parallel_rank_without_picks():
    """A rank whose experts no token picked and without the shared experts
    returns y = 0 (or the residual it was given) on every path."""
    wl = dataclasses.replace(synth.TINY, group=64, T=1, E=64, k=2)
    router = synth.router(wl)
    x, idx_ref, _, _ = gap_resampled_tokens(wl, 1, *router)
    picked = set(idx_ref[0].tolist())
    lo = next(e for e in range(0, wl.E - 4) if not picked & set(range(e, e + 4)))
    L = DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, *router,
                    expert_masters=lambda e: masters(wl, 0, e), expert_range=(lo, lo + 4),
                    with_shared=False)
    for name, (path, _) in PATHS.items():
        y, _, w = run(L, x.cuda(), 1, path)
        assert (w == 0).all() and (y == 0).all(), name
    L.close()


def test_expert_parallel_glm_decode():
    """GLM-5.2 decode layer split over 4 ranks of 64 experts (the shared expert
    on rank 0): partial outputs sum to the whole layer's output."""
    wl = synth.GLM_DECODE
    router = synth.router(wl)
    full = build_layer(wl, router=router)
    ranks = rank_layers(wl, 4, router)
    for step in range(2):
        x, _, _, _ = gap_resampled_tokens(wl, 1, *router, step=step)
        for name in ("fused", "gemv"):
            err = check_partition(wl, full, ranks, x.cuda(), PATHS[name][0], 2e-5)
            print(f"GLM decode, 4 expert ranges, {name}: partial sums vs whole layer {err:.1e}")
    for L in [full] + ranks:
        L.close()
    torch.cuda.empty_cache()
