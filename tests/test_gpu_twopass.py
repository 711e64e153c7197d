"""GPU parity of the two-pass path (COLI_PATH_TWOPASS): a gate/up pass writing h,
h's activation records, a down pass writing each pair's output, the combine.

The arithmetic is the fused kernel's (s8 weight codes, two-digit s8
activations with a power-of-two scale per 256 columns, exact int32 step sums),
so outputs are held to the same norm-wise 2e-3 of the oracle; routing is the
GEMV/GEMM paths' (exact selection).  Units larger than one chunk of 16 pairs,
ragged last chunks, both weight scalings, bf16 tokens, no or two shared
experts, top-p and expert ranges are covered at small sizes against every
output of the oracle; the GLM-5.2 prefill layer against the oracle on sampled
tokens (the busiest expert's included) and against the GEMV path on all."""
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

TOL = 2e-3
TWO = cm.COLI_PATH_TWOPASS


def forward(L, x, T, path=TWO, residual=None):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, L.k), dtype=torch.float32, device="cuda")
    ws = L.workspace(T)
    cm.coli_moe_forward_ex(L.handle, x, T, y, ws, residual=residual, path=path,
                           idx_out=idx, w_out=w)
    torch.cuda.synchronize()
    assert cm.coli_moe_status(L.handle, T, ws) == 0
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def device_x(x, wl):
    return (x.to(torch.bfloat16) if wl.x_dtype == "bf16" else x).cuda().contiguous()


# I a multiple of 256: h has one activation record per 256 columns
BASE = dict(I=256)
VARIANTS = {
    "tiny": {},
    "tiny_gs64": dict(group=64),
    "T1": dict(T=1),
    "T40_gs64": dict(T=40, group=64),
    "T100_tiled_router": dict(T=100, group=64),
    # 75 pairs per expert: five chunks of 16, the last one ragged
    "units_of_five_chunks": dict(T=300, E=8, k=2, group=64),
    "units_of_seven_chunks_per_row": dict(T=200, E=4, k=2),
    "no_shared": dict(n_shared=0, T=70),
    "two_shared": dict(n_shared=2, T=33),
    "k1": dict(k=1, T=50),
    "scale_no_norm": dict(routed_scale=2.5, norm_topk=False, T=20),
    "bf16_x": dict(x_dtype="bf16", group=64, T=65),
    "two_by_three_tiles": dict(H=512, I=768, E=24, k=6, group=64, T=37),
}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_twopass_parity_small(name):
    wl = dataclasses.replace(synth.TINY, **{**BASE, **VARIANTS[name]})
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy(), idx_ref, w_ref)
    L = build_layer(wl, router=(wr, b))
    y, idx, _ = forward(L, device_x(x, wl), wl.T)
    same_selection(idx, idx_ref)
    err = rel_err(y, y_ref)
    assert err <= TOL, err
    # deterministic: no atomics touch the outputs
    y2, _, _ = forward(L, device_x(x, wl), wl.T)
    np.testing.assert_array_equal(y2.view(np.uint32), y.view(np.uint32))
    L.close()


def test_twopass_residual_and_zero_input():
    wl = dataclasses.replace(synth.TINY, I=256, group=64, T=80)
    L = build_layer(wl)
    x = torch.zeros((80, wl.H), dtype=torch.float32, device="cuda")
    y, _, _ = forward(L, x, 80)
    np.testing.assert_array_equal(y, 0.0)
    wr, b = synth.router(wl)
    xr, idx_ref, w_ref, _ = gap_resampled_tokens(wl, 80, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), xr.numpy(), idx_ref, w_ref)
    res = torch.randn((80, wl.H), device="cuda")
    out = res.clone()
    cm.coli_moe_forward_ex(L.handle, xr.cuda(), 80, out, L.workspace(80), residual=out, path=TWO)
    torch.cuda.synchronize()
    assert rel_err(out.cpu().numpy() - res.cpu().numpy(), y_ref) <= TOL
    L.close()


def test_twopass_rejects_what_it_cannot_run():
    wl = dataclasses.replace(synth.TINY, T=70)          # I = 128: not a multiple of 256
    L = build_layer(wl)
    x = torch.randn((70, wl.H), device="cuda")
    y = torch.empty((70, wl.H), device="cuda")
    with pytest.raises(cm.ColiError) as ei:
        cm.coli_moe_forward_ex(L.handle, x, 70, y, L.workspace(70), path=TWO)
    assert ei.value.code == -4   # COLI_E_UNSUPPORTED
    L.close()
    wl8 = dataclasses.replace(synth.TINY, I=256, T=70)
    L8 = build_layer(wl8, bits=8)
    with pytest.raises(cm.ColiError) as ei:
        cm.coli_moe_forward_ex(L8.handle, x, 70, y, L8.workspace(70), path=TWO)
    assert ei.value.code == -4
    L8.close()


@pytest.mark.parametrize("T", [3, 90])
def test_twopass_topp_kept_experts(T):
    """Top-p on the two-pass path: kept sets by the oracle's rule on the same
    weights, outputs against the oracle's forward over the kept experts."""
    wl = dataclasses.replace(synth.TINY, I=256, T=T, group=64, E=32, k=8)
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, T, wr, b)
    L = build_layer(wl, router=(wr, b))
    _, idx_full, w_full = forward(L, x.cuda(), T)
    p = float(np.float32(0.7))           # the value the layer holds (f32)
    cm.coli_moe_layer_set_topp(L.handle, p)
    y, idx, w = forward(L, x.cuda(), T)
    np.testing.assert_array_equal(idx, idx_full)
    keep, _ = oracle.topp_keep(w_full, idx_full, p)
    np.testing.assert_array_equal((w != 0).astype(np.int32), keep)
    wk = w_ref.copy()
    for t in range(T):
        kept = set(idx[t][keep[t] != 0].tolist())
        for j in range(wl.k):
            if int(idx_ref[t, j]) not in kept:
                wk[t, j] = 0.0
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy(), idx_ref, wk)
    assert rel_err(y, y_ref) <= TOL
    L.close()


def test_twopass_expert_ranges_sum_to_the_layer():
    wl = dataclasses.replace(synth.TINY, I=256, T=100, group=64)
    router = synth.router(wl)
    x, _, _, _ = gap_resampled_tokens(wl, wl.T, *router)
    full = build_layer(wl, router=router)
    y_full, _, _ = forward(full, x.cuda(), wl.T)
    parts = []
    for r in range(4):
        L = DeviceLayer(wl.H, wl.I, wl.E, wl.k, wl.n_shared, wl.group, *router,
                        expert_masters=lambda e: masters(wl, 0, e),
                        expert_range=ep.expert_range(wl.E, r, 4),
                        with_shared=r == ep.SHARED_RANK)
        y, _, _ = forward(L, x.cuda(), wl.T)
        parts.append(y.astype(np.float64))
        L.close()
    err = float(np.abs(np.sum(parts, axis=0) - y_full).max() / np.abs(y_full).max())
    assert err <= 2e-5, err
    full.close()


@pytest.fixture(scope="module")
def glm_prefill_layer():
    L = build_layer(synth.GLM_PREFILL)
    yield L
    L.close()
    del L
    torch.cuda.empty_cache()


def test_glm_prefill_two_pass(glm_prefill_layer):
    """Prefill, T = 512 bf16 tokens, gs64, Zipf-skewed routing: every output
    against the f32 GEMV path; against the oracle, all 6144 outputs of tokens
    0, 255 and 511 and of eight tokens routed to the busiest expert (~100
    tokens: seven chunks), the first and last of them included; the shared
    expert's 512 pairs make 32 chunks."""
    wl = synth.GLM_PREFILL
    L = glm_prefill_layer
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    xd = device_x(x, wl)
    y, idx, _ = forward(L, xd, wl.T)
    same_selection(idx, idx_ref)
    y_gemv, _, _ = forward(L, xd, wl.T, path=cm.COLI_PATH_GEMV)
    assert rel_err(y, y_gemv) <= TOL
    experts = OracleExperts(wl)
    xb = x.numpy()
    hot = int(np.argmax(np.bincount(idx_ref.ravel(), minlength=wl.E)))
    hot_toks = np.nonzero((idx_ref == hot).any(1))[0]
    assert hot_toks.size >= 90
    toks = sorted({0, 255, 511} | set(hot_toks[np.linspace(0, hot_toks.size - 1, 8).astype(int)]))
    need = sorted({int(e) for t in toks for e in idx_ref[t]} | {wl.E})
    with cf.ThreadPoolExecutor(16) as ex:
        list(ex.map(experts, need))
    for t in toks:
        y_ref = oracle_tokens(wl, experts, xb[t:t + 1], idx_ref[t:t + 1], w_ref[t:t + 1])
        err = rel_err(y[t:t + 1], y_ref)
        assert err <= TOL, (t, err)
