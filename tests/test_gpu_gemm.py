"""GPU parity of the tensor-core path (tcgen05 grouped GEMM): fp16 operands, f32
accumulation in TMEM.  Outputs within a norm-wise relative error of 1e-2 of the
oracle; routing (done by the same kernels as the GEMV path) exact."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import (OracleExperts, build_layer, gap_resampled_tokens, oracle_tokens,
                             rel_err, same_selection)

pytestmark = pytest.mark.gpu

TOL_TC = 1e-2


def forward(L, x, T, path, residual=None):
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


GEMM_VARIANTS = {
    "tiny": {},
    "tiny_gs64": dict(group=64),
    "T7_gs64": dict(T=7, group=64),
    "two_shared": dict(n_shared=2),
    "k1_fewer_pairs_than_a_box": dict(k=1, n_shared=0, T=9),
    "bf16_x": dict(x_dtype="bf16", group=64),
    "three_row_tiles": dict(H=384, I=256, E=24, k=6, group=64, T=5),
    # units of more than 128 pairs: several N tiles per unit, a ragged last one
    "units_over_128_pairs": dict(T=300, E=8, k=2, group=64),
    "units_over_128_pairs_per_row": dict(T=200, E=4, k=2),
}


@pytest.mark.parametrize("name", list(GEMM_VARIANTS))
def test_gemm_path_parity_small(name):
    wl = dataclasses.replace(synth.TINY, **GEMM_VARIANTS[name])
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy(), idx_ref, w_ref)
    L = build_layer(wl, router=(wr, b))
    y, idx, _ = forward(L, device_x(x, wl), wl.T, cm.COLI_PATH_GEMM)
    same_selection(idx, idx_ref)
    err = rel_err(y, y_ref)
    assert err <= TOL_TC, err
    # deterministic: no atomics touch the outputs
    y2, _, _ = forward(L, device_x(x, wl), wl.T, cm.COLI_PATH_GEMM)
    np.testing.assert_array_equal(y2.view(np.uint32), y.view(np.uint32))


def test_gemm_path_residual_and_zero_input():
    wl = dataclasses.replace(synth.TINY, group=64, T=24)
    L = build_layer(wl)
    x = torch.zeros((24, wl.H), dtype=torch.float32, device="cuda")
    y, _, _ = forward(L, x, 24, cm.COLI_PATH_GEMM)
    np.testing.assert_array_equal(y, 0.0)
    wr, b = synth.router(wl)
    xr, idx_ref, w_ref, _ = gap_resampled_tokens(wl, 24, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), xr.numpy(), idx_ref, w_ref)
    res = torch.randn((24, wl.H), device="cuda")
    out = res.clone()
    cm.coli_moe_forward_ex(L.handle, xr.cuda(), 24, out, L.workspace(24), residual=out,
                           path=cm.COLI_PATH_GEMM)
    torch.cuda.synchronize()
    assert rel_err(out.cpu().numpy() - res.cpu().numpy(), y_ref) <= TOL_TC


def test_gemm_path_at_the_largest_batch():
    """T = 8192, the largest batch a call accepts (16-expert layer): ~2,000
    pairs per expert, so every unit spans many N tiles.  All outputs against
    the f32 GEMV path, 64 sampled tokens against the oracle, selected experts
    exactly."""
    wl = dataclasses.replace(synth.TINY, T=8192, group=64)
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    L = build_layer(wl, router=(wr, b))
    xd = device_x(x, wl)
    y, idx, _ = forward(L, xd, wl.T, cm.COLI_PATH_GEMM)
    same_selection(idx, idx_ref)
    y_gemv, _, _ = forward(L, xd, wl.T, cm.COLI_PATH_GEMV)
    assert rel_err(y, y_gemv) <= TOL_TC
    rows = np.linspace(0, wl.T - 1, 64).astype(int)
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy()[rows], idx_ref[rows], w_ref[rows])
    assert rel_err(y[rows], y_ref) <= TOL_TC


@pytest.fixture(scope="module")
def glm_prefill_layer():
    L = build_layer(synth.GLM_PREFILL)
    yield L
    L.close()
    del L
    torch.cuda.empty_cache()


def test_glm_prefill_tensor_core_path(glm_prefill_layer):
    """Prefill, T = 512 bf16 tokens, gs64, Zipf-skewed routing, 257 resident
    experts.  Every output against the f32 GEMV path (itself held to 2e-3 of the
    oracle); against the oracle, all 6144 outputs of tokens 0, 255 and 511 and
    of eight tokens routed to the busiest expert (~100 tokens: its units span
    two N tiles), the first and last of them included."""
    wl = synth.GLM_PREFILL
    L = glm_prefill_layer
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    xd = device_x(x, wl)
    y, idx, _ = forward(L, xd, wl.T, cm.COLI_PATH_GEMM)
    same_selection(idx, idx_ref)
    y_gemv, _, _ = forward(L, xd, wl.T, cm.COLI_PATH_GEMV)
    assert rel_err(y, y_gemv) <= TOL_TC
    import concurrent.futures as cf
    experts = OracleExperts(wl)
    xb = x.numpy()            # already bf16-representable: the device reads the same values
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
        assert err <= TOL_TC, (t, err)
