"""GPU parity: libcolimoe (through the C ABI) against the CPU oracle on the same
seeded inputs.  Bit-exact for container bytes, scales, dequantised weights,
selected expert sets and union lists; layer outputs within a norm-wise relative
error of 2e-3 on the small-batch paths (GEMV: fp16 digits, f32 accumulation;
FUSED: s8 digits, exact int32 step sums, f32 across steps)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import (OracleExperts, build_layer, gap_resampled_tokens, masters,
                             oracle_tokens, ordered_ok, rel_err, same_selection)

pytestmark = pytest.mark.gpu

TOL_F32 = 2e-3


def forward(L, x, T, path=cm.COLI_PATH_GEMV, residual=None):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, L.k), dtype=torch.float32, device="cuda")
    ws = L.workspace(T)
    cm.coli_moe_forward_ex(L.handle, x, T, y, ws, residual=residual, path=path,
                           idx_out=idx, w_out=w)
    torch.cuda.synchronize()
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def check_weights(idx, w, idx_ref, w_ref):
    oi, orf = np.argsort(idx, 1), np.argsort(idx_ref, 1)
    np.testing.assert_allclose(np.take_along_axis(w, oi, 1),
                               np.take_along_axis(w_ref, orf, 1), rtol=2e-6, atol=1e-7)


def device_x(x, wl):
    return (x.to(torch.bfloat16) if wl.x_dtype == "bf16" else x).cuda().contiguous()


# ---------------------------------------------------------------------------
# container on the device
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("group", [0, 64])
@pytest.mark.parametrize("shape", [(256, 128), (6144, 2048)])
def test_device_quantizer_matches_host_packer(group, shape):
    H, I = shape
    wl = dataclasses.replace(synth.TINY, H=H, I=I, group=group)
    g, u, d = masters(wl, 0, 3)
    blob = torch.empty(cm.coli_moe_expert_bytes(H, I, group), dtype=torch.uint8, device="cuda")
    cm.coli_moe_quantize_expert_device(H, I, group, g, u, d, blob)
    cont = []
    for m in (g, u, d):
        cont += list(oracle.quantize(m.cpu().numpy(), group))
    host = cm.coli_moe_pack_expert(H, I, group, *cont)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(blob.cpu().numpy(), host)


@pytest.mark.parametrize("group", [0, 64])
@pytest.mark.parametrize("shape", [(256, 128), (6144, 2048)])
def test_fp8_block_requantisation_matches_host(group, shape):
    """FP8 E4M3 experts with 128 x 128 block scales -> int4 container on the
    device, byte for byte what the oracle's FP8 decode followed by the host
    quantiser and packer give."""
    H, I = shape
    rng = np.random.default_rng(11 + group)

    def fp8(R, K):
        codes = rng.integers(0, 256, (R, K), dtype=np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x3C              # finite codes only
        bs = rng.uniform(1e-4, 4e-4, ((R + 127) // 128, (K + 127) // 128)).astype(np.float32)
        return codes, bs

    mats = [fp8(I, H), fp8(I, H), fp8(H, I)]
    cont = []
    for codes, bs in mats:
        cont += list(oracle.quantize(oracle.fp8_block_dequant(codes, bs), group))
    host = cm.coli_moe_pack_expert(H, I, group, *cont)
    dev = [(torch.from_numpy(c).cuda(), torch.from_numpy(b).cuda()) for c, b in mats]
    blob = torch.empty(cm.coli_moe_expert_bytes(H, I, group), dtype=torch.uint8, device="cuda")
    cm.coli_moe_quantize_expert_fp8_device(H, I, group, dev[0][0], dev[1][0], dev[2][0],
                                           dev[0][1], dev[1][1], dev[2][1], blob)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(blob.cpu().numpy(), host)


@pytest.mark.parametrize("group", [0, 64])
def test_dequant_bit_exact(group):
    wl = dataclasses.replace(synth.TINY, group=group)
    L = build_layer(wl)
    ref = OracleExperts(wl)
    for e in (0, 7, wl.E):              # routed and shared
        for which in range(3):
            R, K = (wl.I, wl.H) if which < 2 else (wl.H, wl.I)
            out = torch.empty((R, K), dtype=torch.float32, device="cuda")
            cm.coli_moe_dequant_debug(L.handle, e, which, out)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32),
                                          ref(e)[which].view(np.uint32))


# ---------------------------------------------------------------------------
# routing and union
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,xdt", [(4, "f32"), (1, "f32"), (40, "f32"), (33, "bf16"),
                                   (512, "bf16")])
def test_route_glm_router(T, xdt):
    wl = dataclasses.replace(synth.GLM_DECODE, x_dtype=xdt)
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, T, wr, b)
    L = build_layer(dataclasses.replace(synth.TINY, H=wl.H, E=wl.E, k=wl.k),
                    router=(wr, b))
    idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    cm.coli_moe_route(L.handle, device_x(x, wl), T, idx, w, L.workspace(T))
    torch.cuda.synchronize()
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    same_selection(idx, idx_ref, ordered_ok(x.numpy(), wr.numpy(), b.numpy(), idx_ref, wl.k))
    check_weights(idx, w, idx_ref, w_ref)


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (3, 8, 256), (37, 4, 16), (512, 8, 256),
                                   (2048, 8, 256), (5, 1, 1), (64, 32, 1024)])
def test_union_matches_oracle(T, k, E):
    rng = np.random.default_rng(T * 1000 + E)
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.1
    idx = np.stack([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)])
    idx = idx.astype(np.int32)
    ref = oracle.union(idx, E)
    d = {n: torch.full((s,), -7, dtype=torch.int32, device="cuda") for n, s in
         (("offsets", E + 1), ("pair_tok", T * k), ("pair_slot", T * k), ("uniq", E),
          ("n_uniq", 1))}
    cm.coli_moe_union(torch.from_numpy(idx).cuda(), T, k, E, d["offsets"], d["pair_tok"],
                      d["pair_slot"], d["uniq"], d["n_uniq"])
    torch.cuda.synchronize()
    n = int(d["n_uniq"].item())
    assert n == ref[4]
    np.testing.assert_array_equal(d["offsets"].cpu().numpy(), ref[0])
    np.testing.assert_array_equal(d["pair_tok"].cpu().numpy(), ref[1])
    np.testing.assert_array_equal(d["pair_slot"].cpu().numpy(), ref[2])
    np.testing.assert_array_equal(d["uniq"].cpu().numpy()[:n], ref[3])
    assert np.all(d["uniq"].cpu().numpy()[n:] == -7)     # untouched past n_uniq


# ---------------------------------------------------------------------------
# whole layer, small shapes (every output element against the oracle)
# ---------------------------------------------------------------------------

VARIANTS = {
    "tiny": {},
    "tiny_gs64": dict(group=64),
    "T1": dict(T=1),
    "T7_gs64": dict(T=7, group=64),
    "T40_tiled_router": dict(T=40),
    "T64_chunked_units": dict(T=64, E=8, k=2, group=64),
    "no_shared": dict(n_shared=0),
    "two_shared": dict(n_shared=2),
    "k1": dict(k=1),
    "E_eq_k": dict(E=4, k=4),
    "scale_no_norm": dict(routed_scale=2.5, norm_topk=False),
    "bf16_x": dict(x_dtype="bf16", group=64),
    "three_tiles": dict(H=384, I=256, E=24, k=6, group=64, T=5),
    "skewed_many_tokens": dict(T=96, E=8, k=2, group=64),
}


SMALL_PATHS = {"gemv": cm.COLI_PATH_GEMV, "fused": cm.COLI_PATH_FUSED}


def fused_applies(wl, T):
    return (T <= 64 and T * (wl.k + wl.n_shared) <= 640 and wl.E <= 256 and wl.k <= 32
            and wl.n_shared <= 4 and wl.H % 256 == 0 and wl.I <= 4096)


@pytest.mark.parametrize("path", list(SMALL_PATHS))
@pytest.mark.parametrize("name", list(VARIANTS))
def test_layer_parity_small(name, path):
    wl = dataclasses.replace(synth.TINY, **VARIANTS[name])
    if path == "fused" and not fused_applies(wl, wl.T):
        pytest.skip("outside the fused kernel's limits (covered by the rejection test)")
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy(), idx_ref, w_ref)
    L = build_layer(wl, router=(wr, b))
    y, idx, w = forward(L, device_x(x, wl), wl.T, path=SMALL_PATHS[path])
    same_selection(idx, idx_ref, ordered_ok(x.numpy(), wr.numpy(), b.numpy(), idx_ref, wl.k))
    check_weights(idx, w, idx_ref, w_ref)
    err = rel_err(y, y_ref)
    assert err <= TOL_F32, err
    # deterministic: a second run gives the same bytes
    y2, _, _ = forward(L, device_x(x, wl), wl.T, path=SMALL_PATHS[path])
    np.testing.assert_array_equal(y2.view(np.uint32), y.view(np.uint32))


@pytest.mark.parametrize("path", list(SMALL_PATHS))
def test_residual_and_zero_input(path):
    wl = dataclasses.replace(synth.TINY, group=64)
    L = build_layer(wl)
    x = torch.zeros((3, wl.H), dtype=torch.float32, device="cuda")
    y, _, _ = forward(L, x, 3, path=SMALL_PATHS[path])
    np.testing.assert_array_equal(y, 0.0)          # x = 0 -> y = 0 exactly
    wr, b = synth.router(wl)
    xr, idx_ref, w_ref, _ = gap_resampled_tokens(wl, 4, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), xr.numpy(), idx_ref, w_ref)
    res = torch.randn((4, wl.H), device="cuda")
    out = res.clone()
    cm.coli_moe_forward_ex(L.handle, xr.cuda(), 4, out, L.workspace(4), residual=out,
                           path=SMALL_PATHS[path])
    torch.cuda.synchronize()
    assert rel_err(out.cpu().numpy() - res.cpu().numpy(), y_ref) <= TOL_F32


def test_fused_rejects_sizes_outside_its_limits():
    wl = dataclasses.replace(synth.TINY, T=65)
    L = build_layer(wl)
    x = torch.randn((65, wl.H), device="cuda")
    y = torch.empty((65, wl.H), device="cuda")
    with pytest.raises(cm.ColiError) as ei:
        cm.coli_moe_forward_ex(L.handle, x, 65, y, L.workspace(65), path=cm.COLI_PATH_FUSED)
    assert ei.value.code == -4   # COLI_E_UNSUPPORTED


@pytest.mark.parametrize("T", [1, 5, 16, 33, 64])
def test_auto_small_batches_equal_fused(T):
    """AUTO picks the fused kernel for small batches: same bytes as asking for it."""
    wl = dataclasses.replace(synth.TINY, T=T, group=64)
    L = build_layer(wl)
    x = torch.randn((T, wl.H), device="cuda")
    ya, _, _ = forward(L, x, T, path=cm.COLI_PATH_AUTO)
    yf, _, _ = forward(L, x, T, path=cm.COLI_PATH_FUSED)
    np.testing.assert_array_equal(ya.view(np.uint32), yf.view(np.uint32))


def test_rmsnorm_matches_oracle():
    x = torch.randn((5, 6144), device="cuda") * 3
    out = torch.empty_like(x)
    cm.coli_moe_rmsnorm(x, 5, 6144, 1e-5, out)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(x.cpu().numpy(), 1e-5)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=2e-6, atol=1e-7)


# ---------------------------------------------------------------------------
# GLM-5.2-shaped layers at full size
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def glm_decode_layer():
    L = build_layer(synth.GLM_DECODE)
    yield L
    L.close()
    del L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", list(SMALL_PATHS))
def test_glm_decode_full_layer(glm_decode_layer, path):
    """Decode, T = 1, per-row scales, 257 resident experts: all 6144 outputs."""
    wl = synth.GLM_DECODE
    L = glm_decode_layer
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    experts = OracleExperts(wl)
    for step in range(2):
        x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, 1, wr, b, step=step)
        y, idx, w = forward(L, x.cuda(), 1, path=SMALL_PATHS[path])
        same_selection(idx, idx_ref)
        check_weights(idx, w, idx_ref, w_ref)
        y_ref = oracle_tokens(wl, experts, x.numpy(), idx_ref, w_ref)
        err = rel_err(y, y_ref)
        assert err <= TOL_F32, err


@pytest.mark.parametrize("path", list(SMALL_PATHS))
def test_glm_gemv_batch_over_staging_cap(glm_decode_layer, path):
    """A batch of 16 tokens at full size: on the GEMV path more tokens than one
    pass stages in shared memory, so units of several pairs run several passes;
    on the fused path the largest column-group count (16 pairs per unit).
    Selection of all tokens exact; two tokens' outputs against the oracle."""
    wl = synth.GLM_DECODE
    L = glm_decode_layer
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, 16, wr, b, step=7)
    y, idx, w = forward(L, x.cuda(), 16, path=SMALL_PATHS[path])
    same_selection(idx, idx_ref)
    check_weights(idx, w, idx_ref, w_ref)
    experts = OracleExperts(wl)
    for t in (0, 15):
        y_ref = oracle_tokens(wl, experts, x.numpy()[t:t + 1], idx_ref[t:t + 1], w_ref[t:t + 1])
        err = rel_err(y[t:t + 1], y_ref)
        assert err <= TOL_F32, (t, err)
        experts.cache.clear()


@pytest.fixture(scope="module")
def glm_mtp_layer():
    L = build_layer(synth.GLM_MTP)
    yield L
    L.close()
    del L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", list(SMALL_PATHS))
def test_glm_mtp_verify_steps(glm_mtp_layer, path):
    """MTP verify: 64 steps of 3 positions, gs64.  Every step's selection and union
    is checked exactly; outputs of two steps are checked element by element."""
    wl = synth.GLM_MTP
    L = glm_mtp_layer
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    experts = OracleExperts(wl)
    for step in range(wl.steps):
        x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b, step=step)
        y, idx, w = forward(L, x.cuda(), wl.T, path=SMALL_PATHS[path])
        same_selection(idx, idx_ref)
        ref = oracle.union(idx_ref, wl.E)
        d = {n: torch.empty((s,), dtype=torch.int32, device="cuda") for n, s in
             (("o", wl.E + 1), ("t", wl.T * wl.k), ("s", wl.T * wl.k), ("u", wl.E), ("n", 1))}
        cm.coli_moe_union(torch.from_numpy(idx).cuda(), wl.T, wl.k, wl.E, d["o"], d["t"],
                          d["s"], d["u"], d["n"])
        torch.cuda.synchronize()
        assert int(d["n"].item()) == ref[4]
        np.testing.assert_array_equal(d["o"].cpu().numpy(), ref[0])
        np.testing.assert_array_equal(d["t"].cpu().numpy(), ref[1])
        if step in (0, wl.steps - 1):
            y_ref = oracle_tokens(wl, experts, x.numpy(), idx_ref, w_ref)
            err = rel_err(y, y_ref)
            assert err <= TOL_F32, err
            experts.cache.clear()


# ---------------------------------------------------------------------------
# activations with outlier channels and a wide dynamic range
# ---------------------------------------------------------------------------

def outlier_tokens(wl, wr, b, step, max_rounds=64):
    """Four tokens on N(0, 1) draws: (0) one channel at 100x, (1) four channels
    at 1000x, (2) magnitudes 2^u, u uniform in [-10, 10], random signs,
    (3) sixteen channels at 100x; each then scaled to unit RMS, as a normalised
    layer input is (the ratios between channels are what the activation
    encodings must carry; the router keeps its usual operating range).
    Positions and signs come from a seeded generator; a token whose oracle gap
    is under 1e-3 is drawn again."""
    wr_np, b_np = wr.cpu().numpy(), b.cpu().numpy()
    out = []
    for case in range(4):
        for r in range(max_rounds):
            rng = np.random.default_rng([wl.seed, step, case, r])
            x = synth.tokens(wl, 1, 0, 1000 + 97 * step + case, [r]).numpy()[0].copy()
            if case == 2:
                x = np.where(rng.random(wl.H) < 0.5, -1.0, 1.0) * np.exp2(rng.uniform(-10, 10, wl.H))
            else:
                n, amp = {0: (1, 100.0), 1: (4, 1000.0), 3: (16, 100.0)}[case]
                pos = rng.choice(wl.H, n, replace=False)
                x[pos] = amp * np.where(rng.random(n) < 0.5, -1.0, 1.0)
            x = (x / np.sqrt(np.mean(np.square(x, dtype=np.float64)))).astype(np.float32)[None]
            idx, w, gap = oracle.route(x, wr_np, b_np, wl.k, wl.routed_scale, wl.norm_topk)
            if gap[0] >= 1e-3:
                out.append((x[0], idx[0], w[0]))
                break
        else:
            raise RuntimeError("gap rule did not converge")
    return (np.stack([o[0] for o in out]), np.stack([o[1] for o in out]),
            np.stack([o[2] for o in out]))


def per_element_error(y, ref):
    """max |y - ref| / max(|ref|, 1e-6 max |ref|), element by element (reported)."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    floor = 1e-6 * np.abs(ref).max()
    return float((np.abs(y - ref) / np.maximum(np.abs(ref), floor)).max())


OUTLIER_PATHS = {"fused": (cm.COLI_PATH_FUSED, TOL_F32), "gemv": (cm.COLI_PATH_GEMV, TOL_F32),
                 "gemm": (cm.COLI_PATH_GEMM, 1e-2)}


def check_outliers(wl, L, step):
    import concurrent.futures as cf
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    x, idx_ref, w_ref = outlier_tokens(wl, wr, b, step)
    experts = OracleExperts(wl)
    need = sorted({int(e) for e in idx_ref.ravel()} | {wl.E + s for s in range(wl.n_shared)})
    with cf.ThreadPoolExecutor(8) as ex:
        list(ex.map(experts, need))
    y_ref = oracle_tokens(wl, experts, x, idx_ref, w_ref)
    xd = torch.from_numpy(x).cuda()
    for name, (path, tol) in OUTLIER_PATHS.items():
        y, idx, _ = forward(L, xd, 4, path=path)
        same_selection(idx, idx_ref)
        for t in range(4):
            err = rel_err(y[t], y_ref[t])
            print(f"{wl.name} {name} token {t}: norm-wise {err:.2e}, "
                  f"per-element {per_element_error(y[t], y_ref[t]):.2e}")
            assert err <= tol, (name, t, err)
    for t in range(4):   # the one-token fused path
        y, _, _ = forward(L, xd[t:t + 1].contiguous(), 1, path=cm.COLI_PATH_FUSED)
        assert rel_err(y[0], y_ref[t]) <= TOL_F32, t


def test_outlier_activations_per_row(glm_decode_layer):
    check_outliers(synth.GLM_DECODE, glm_decode_layer, step=0)


def test_outlier_activations_gs64(glm_mtp_layer):
    check_outliers(synth.GLM_MTP, glm_mtp_layer, step=1)
