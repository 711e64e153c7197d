"""GPU parity of the layer stack (coli_moe_stack_forward): x <- x + MoE_l(RMSNorm(x))
for l = 0 .. L-1, against the CPU oracle, teacher-forced layer by layer.

For every layer l the oracle takes the GPU's layer-l input x_l, normalises it
(orc_rmsnorm), routes it (orc_route) and runs the routed and shared experts
(orc_token_forward); the GPU's x_{l+1} must equal x_l + that output within the
path's tolerance.  Routing is compared bit-exactly on every token whose oracle
gap sel_(k) - sel_(k+1) is at least 1e-3; tokens below that gap (the gap can
only be enforced by redrawing the stack's input, i.e. at layer 0) are excluded
and counted.  The stack call itself is checked to give the same bytes as the
layer-by-layer calls whose intermediate states feed the oracle.

Configuration: the stack of GLM-5.2-shaped layers (hidden 6144, 256 routed + 1
shared expert, intermediate 2048, top-8, int4 with one scale per 64 columns,
RMSNorm eps 1e-5 with unit gain, residual add), and a 3-layer stack of the tiny
layer shape on every path.
"""
import concurrent.futures as cf
import dataclasses
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import OracleExperts, build_layer

pytestmark = pytest.mark.gpu

TOL = {cm.COLI_PATH_FUSED: 2e-3, cm.COLI_PATH_GEMV: 2e-3, cm.COLI_PATH_GEMM: 1e-2,
       cm.COLI_PATH_TWOPASS: 2e-3}
THREADS = max(1, min(16, os.cpu_count() or 1))


def stack_tokens(wl, T, step=0, max_rounds=64):
    """x_0 [T, H] f32 whose RMSNorm meets the gap rule at layer 0's router."""
    wr, b = synth.router(wl, 0)
    redraw = [0] * T
    for _ in range(max_rounds):
        x = synth.tokens(wl, T, 0, step, redraw)
        _, _, gap = oracle.route(oracle.rmsnorm(x.numpy(), wl.eps), wr.numpy(), b.numpy(),
                                 wl.k, wl.routed_scale, wl.norm_topk)
        bad = np.nonzero(gap < 1e-3)[0]
        if bad.size == 0:
            return x
        for t in bad:
            redraw[t] += 1
    raise RuntimeError("gap rule did not converge")


def oracle_moe(wl, layer, xn, idx, w, tokens):
    """Oracle MoE outputs (float64 of the f32 result) of the given tokens of one
    layer; the experts they need are dequantised in parallel threads first."""
    experts = OracleExperts(wl, layer)
    need = sorted({int(e) for t in tokens for e in idx[t]} |
                  {wl.E + s for s in range(wl.n_shared)})
    with cf.ThreadPoolExecutor(THREADS) as ex:
        list(ex.map(experts, need))
        outs = list(ex.map(
            lambda t: oracle.token_forward(
                xn[t], w[t], [experts(int(e)) for e in idx[t]] +
                [experts(wl.E + s) for s in range(wl.n_shared)], wl.n_shared),
            tokens))
    return np.stack(outs).astype(np.float64)


def run_stack(handles, x0, T, eps, path):
    """(x after the whole stack call, [x_0 .. x_L] from one call per layer)."""
    ws = torch.empty(cm.coli_moe_stack_workspace_size(handles, T), dtype=torch.uint8,
                     device="cuda")
    xf = x0.clone()
    cm.coli_moe_stack_forward(handles, xf, T, eps, ws, path=path)
    xs = [x0.clone()]
    for h in handles:
        xl = xs[-1].clone()
        cm.coli_moe_stack_forward([h], xl, T, eps, ws, path=path)
        xs.append(xl)
    torch.cuda.synchronize()
    return xf, xs


def check_stack(wl, layers, x0, path, sample=None):
    """Teacher-forced parity of every layer; returns (worst error, excluded tokens:
    those under the gap whose GPU selection differs from the oracle's)."""
    T, H, eps = x0.shape[0], wl.H, wl.eps
    handles = [L.handle for L in layers]
    xf, xs = run_stack(handles, x0, T, eps, path)
    np.testing.assert_array_equal(xf.cpu().numpy().view(np.uint32),
                                  xs[-1].cpu().numpy().view(np.uint32))
    worst, excluded = 0.0, 0
    for l, L in enumerate(layers):
        x_l = xs[l].cpu().numpy()
        # the GPU's own routing of this layer: the stack's two steps for one layer
        xn = torch.empty_like(xs[l])
        cm.coli_moe_rmsnorm(xs[l], T, H, eps, xn)
        y = xs[l].clone()
        idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
        cm.coli_moe_forward_ex(L.handle, xn, T, y, L.workspace(T), residual=y, path=path,
                               idx_out=idx)
        torch.cuda.synchronize()
        y = y.cpu().numpy()
        np.testing.assert_array_equal(y.view(np.uint32), xs[l + 1].cpu().numpy().view(np.uint32))
        xn_ref = oracle.rmsnorm(x_l, eps)
        np.testing.assert_allclose(xn.cpu().numpy(), xn_ref, rtol=2e-6, atol=1e-7)
        wr, b = L.router_w.cpu().numpy(), L.router_b.cpu().numpy()
        idx_ref, w_ref, gap = oracle.route(xn_ref, wr, b, wl.k, wl.routed_scale, wl.norm_topk)
        idx = idx.cpu().numpy()
        same = (np.sort(idx, 1) == np.sort(idx_ref, 1)).all(1)
        wide = gap >= 1e-3
        np.testing.assert_array_equal(np.sort(idx[wide], 1), np.sort(idx_ref[wide], 1))
        # a token under the gap whose selection still agrees is checked as well;
        # one whose selection differs is excluded and counted
        ok = wide | same
        excluded += int((~ok).sum())
        toks = [t for t in (range(T) if sample is None else sample(l, idx)) if ok[t]]
        if not toks:
            continue
        moe = oracle_moe(wl, l, xn_ref, idx_ref, w_ref, toks)
        y_ref = (x_l[toks].astype(np.float64) + moe).astype(np.float32)
        err = float(np.abs(y[toks] - y_ref).max() / max(np.abs(moe).max(), 1e-30))
        assert err <= TOL[path], (l, err)
        worst = max(worst, err)
    return worst, excluded


# ---------------------------------------------------------------------------
# tiny shape, 3 layers, every path
# ---------------------------------------------------------------------------

TINY_STACK = dataclasses.replace(synth.TINY, group=64, layers=3, seed=5101)


@pytest.fixture(scope="module")
def tiny_stack():
    layers = [build_layer(TINY_STACK, layer=l) for l in range(TINY_STACK.layers)]
    yield layers
    for L in layers:
        L.close()


@pytest.mark.parametrize("T", [1, 4, 50])
@pytest.mark.parametrize("path", [cm.COLI_PATH_FUSED, cm.COLI_PATH_GEMV, cm.COLI_PATH_GEMM])
def test_tiny_stack_teacher_forced(tiny_stack, path, T):
    x0 = stack_tokens(TINY_STACK, T, step=T).cuda()
    worst, excluded = check_stack(TINY_STACK, tiny_stack, x0, path)
    print(f"tiny stack path {path} T={T}: worst layer error {worst:.2e}, "
          f"excluded tokens {excluded}")
    assert excluded <= T * TINY_STACK.layers // 2


# the two-pass path needs I to be a multiple of 256
TINY_STACK_I256 = dataclasses.replace(TINY_STACK, I=256, seed=5102)


@pytest.fixture(scope="module")
def tiny_stack_i256():
    layers = [build_layer(TINY_STACK_I256, layer=l) for l in range(TINY_STACK_I256.layers)]
    yield layers
    for L in layers:
        L.close()


@pytest.mark.parametrize("T", [3, 90])
def test_tiny_stack_two_pass(tiny_stack_i256, T):
    x0 = stack_tokens(TINY_STACK_I256, T, step=200 + T).cuda()
    worst, excluded = check_stack(TINY_STACK_I256, tiny_stack_i256, x0, cm.COLI_PATH_TWOPASS)
    print(f"tiny stack two-pass T={T}: worst layer error {worst:.2e}, excluded tokens {excluded}")
    assert excluded <= T * TINY_STACK_I256.layers // 2


def test_tiny_stack_auto_takes_two_pass_past_the_fused_limit(tiny_stack_i256):
    handles = [L.handle for L in tiny_stack_i256]
    x0 = stack_tokens(TINY_STACK_I256, 90, step=390).cuda()
    a, _ = run_stack(handles, x0, 90, TINY_STACK_I256.eps, cm.COLI_PATH_AUTO)
    b, _ = run_stack(handles, x0, 90, TINY_STACK_I256.eps, cm.COLI_PATH_TWOPASS)
    np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))


def test_tiny_stack_auto_equals_chosen_path(tiny_stack):
    """AUTO takes the fused kernel at 4 tokens and the tensor-core path at 80:
    the same bytes as asking for those paths."""
    handles = [L.handle for L in tiny_stack]
    for T, path in ((4, cm.COLI_PATH_FUSED), (80, cm.COLI_PATH_GEMM)):
        x0 = stack_tokens(TINY_STACK, T, step=100 + T).cuda()
        a, _ = run_stack(handles, x0, T, TINY_STACK.eps, cm.COLI_PATH_AUTO)
        b, _ = run_stack(handles, x0, T, TINY_STACK.eps, path)
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32),
                                      b.cpu().numpy().view(np.uint32))


# ---------------------------------------------------------------------------
# GLM-5.2 shape, 16 layers (87.3 GB of int4 gs64 experts resident)
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def glm_stack():
    wl = synth.GLM_STACK
    layers = [build_layer(wl, layer=l) for l in range(wl.layers)]
    yield layers
    for L in layers:
        L.close()
    del layers
    torch.cuda.empty_cache()


def free_running_error(wl, layers, x0, x_gpu):
    """Information only: the oracle's own 16-layer chain from x_0 against the GPU."""
    x = x0.cpu().numpy()
    for l, L in enumerate(layers):
        xn = oracle.rmsnorm(x, wl.eps)
        idx, w, _ = oracle.route(xn, L.router_w.cpu().numpy(), L.router_b.cpu().numpy(),
                                 wl.k, wl.routed_scale, wl.norm_topk)
        x = (x.astype(np.float64) + oracle_moe(wl, l, xn, idx, w, range(x.shape[0]))
             ).astype(np.float32)
    return float(np.abs(x_gpu - x).max() / np.abs(x).max())


def test_glm_stack16_decode_all_outputs(glm_stack):
    """One token through all 16 layers (fused path): every layer's 6144 outputs."""
    wl = synth.GLM_STACK
    x0 = stack_tokens(wl, 1, step=0).cuda()
    worst, excluded = check_stack(wl, glm_stack, x0, cm.COLI_PATH_FUSED)
    _, xs = run_stack([L.handle for L in glm_stack], x0, 1, wl.eps, cm.COLI_PATH_FUSED)
    info = free_running_error(wl, glm_stack, x0, xs[-1].cpu().numpy())
    print(f"GLM stack T=1: worst layer error {worst:.2e}, excluded {excluded}, "
          f"free-running error after 16 layers {info:.2e} (information)")
    assert excluded <= wl.layers // 2


def test_glm_stack16_sixteen_tokens(glm_stack):
    """16 tokens (fused path), two tokens per layer against the oracle, the
    selection of all 16 compared on every layer."""
    wl = synth.GLM_STACK
    x0 = stack_tokens(wl, 16, step=1).cuda()
    worst, excluded = check_stack(wl, glm_stack, x0, cm.COLI_PATH_FUSED,
                                  sample=lambda l, idx: (l % 16, (l + 7) % 16))
    print(f"GLM stack T=16: worst layer error {worst:.2e}, excluded {excluded}")
    assert excluded <= 16 * wl.layers // 2


def test_glm_stack16_prefill_two_pass(glm_stack):
    """512 tokens on the two-pass path (what AUTO takes there): the same samples
    as the tensor-core test below, at the s8 path's tolerance."""
    wl = synth.GLM_STACK

    def sample(l, idx):
        counts = np.bincount(idx.ravel(), minlength=wl.E)
        hot = int(np.argmax(counts))
        last_hot = int(np.nonzero((idx == hot).any(1))[0][-1])
        return (last_hot, 256 + (37 * l) % 256)

    x0 = stack_tokens(wl, 512, step=2).cuda()
    worst, excluded = check_stack(wl, glm_stack, x0, cm.COLI_PATH_TWOPASS, sample=sample)
    print(f"GLM stack T=512 two-pass: worst layer error {worst:.2e}, excluded {excluded}")
    assert excluded <= 512 * wl.layers // 2


def test_glm_stack16_prefill_tensor_cores(glm_stack):
    """512 tokens (tensor-core path): on every layer the last token routed to
    the layer's busiest expert (the expert whose tokens fill the most N-tile
    columns) and one token past the first 256; every token's selection."""
    wl = synth.GLM_STACK

    def sample(l, idx):
        counts = np.bincount(idx.ravel(), minlength=wl.E)
        hot = int(np.argmax(counts))
        last_hot = int(np.nonzero((idx == hot).any(1))[0][-1])
        return (last_hot, 256 + (37 * l) % 256)

    x0 = stack_tokens(wl, 512, step=2).cuda()
    worst, excluded = check_stack(wl, glm_stack, x0, cm.COLI_PATH_GEMM, sample=sample)
    print(f"GLM stack T=512: worst layer error {worst:.2e}, excluded {excluded}")
    assert excluded <= 512 * wl.layers // 2
