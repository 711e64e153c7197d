"""Pins for the CPU oracle: hand-worked examples, closed forms, invariants and
special cases that reduce to library routines.  None of these re-types the
oracle's own formulas; each one fails for a plausible slip (dropped term, wrong
sign or index, transposed operand, wrong rounding mode)."""
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _records(name):
    recs, cur = [], {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            if key in cur:
                recs.append(cur)
                cur = {}
            cur[key] = val.strip()
    if cur:
        recs.append(cur)
    return recs


def _floats(s):
    return np.array([float(v) for v in s.split()], np.float32)


# --------------------------------------------------------------------------
# container: quantise / dequantise
# --------------------------------------------------------------------------

def test_quant_hand_examples():
    recs = _records("quant_examples.txt")
    assert len(recs) == 4
    for r in recs:
        row = _floats(r["row"])[None, :]
        packed, scales = oracle.quantize(row, 0)
        assert scales[0, 0] == np.float32(float(r["scale"]))
        assert packed[0].tobytes().hex() == "".join(r["bytes"].split())
        deq = oracle.dequantize(packed, scales, row.shape[1], 0)
        np.testing.assert_array_equal(deq[0], _floats(r["dequant"]))
        # codes follow from dequant / scale for the nonzero-scale rows
        if scales[0, 0] != 0:
            np.testing.assert_array_equal(np.rint(deq[0] / scales[0, 0]),
                                          _floats(r["codes"]))


def test_dequant_every_byte():
    """Brute force over all 256 bytes: low nibble = even column, two's complement."""
    packed = np.arange(256, dtype=np.uint8)[:, None]
    scales = np.full((256, 1), 0.25, np.float32)
    deq = oracle.dequantize(packed, scales, 2, 0)
    sext = lambda n: n - 16 if n >= 8 else n
    want = np.array([[sext(b & 15), sext(b >> 4)] for b in range(256)], np.float32) * 0.25
    np.testing.assert_array_equal(deq, want)


def test_quant_codes_pairs_roundtrip():
    """Every pair of codes in [-7, 7] survives quantise(dequantise) exactly when the
    row also holds the +-7 code that fixes the scale."""
    s = np.float32(0.0390625)
    for a in range(-7, 8):
        for b in range(-7, 8):
            q = np.array([a, b, 7, 0], np.float32)
            row = (q * s)[None, :]
            packed, scales = oracle.quantize(row, 0)
            assert scales[0, 0] == s
            deq = oracle.dequantize(packed, scales, 4, 0)
            np.testing.assert_array_equal(deq[0], row[0])


@pytest.mark.parametrize("group", [0, 64])
def test_quant_error_bound_and_roundtrip(group):
    """|w - w'| <= s/2 (rounding to nearest), max element hits +-7, and the
    container is a fixed point: re-quantising w' gives the same bytes and scales."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((300, 256)) * 0.02).astype(np.float32)
    w[5] = 0.0                                   # a zero row
    packed, scales = oracle.quantize(w, group)
    deq = oracle.dequantize(packed, scales, 256, group)
    gs = 256 if group == 0 else group
    s_full = np.repeat(scales, gs, axis=1)
    err = np.abs(w.astype(np.float64) - deq.astype(np.float64))
    assert np.all(err <= s_full.astype(np.float64) * 0.5 * (1 + 1e-6) + 1e-12)
    np.testing.assert_array_equal(deq[5], 0.0)
    # the group maximum is coded as +-7
    q = np.rint(deq / np.where(s_full == 0, 1, s_full))
    qg = np.abs(q).reshape(300, -1, gs).max(axis=2)
    assert np.all(qg[np.arange(300) != 5] == 7)
    p2, s2 = oracle.quantize(deq, group)
    np.testing.assert_array_equal(p2, packed)
    np.testing.assert_array_equal(s2, scales)


def test_group_reduces_to_per_row():
    """When every 64-column group has the same max |w|, gs64 and per-row coincide."""
    rng = np.random.default_rng(3)
    w = rng.uniform(-0.5, 0.5, (16, 256)).astype(np.float32)
    w[:, ::64] = 0.75
    p0, s0 = oracle.quantize(w, 0)
    p1, s1 = oracle.quantize(w, 64)
    np.testing.assert_array_equal(p0, p1)
    np.testing.assert_array_equal(s1, np.repeat(s0, 4, axis=1))


def test_quant_rejects_bad_shapes():
    with pytest.raises(RuntimeError):
        oracle.quantize(np.zeros((2, 3), np.float32), 0)      # odd columns
    with pytest.raises(RuntimeError):
        oracle.quantize(np.zeros((2, 96), np.float32), 64)    # not a multiple of 64


# --------------------------------------------------------------------------
# router
# --------------------------------------------------------------------------

def test_router_hand_examples():
    for r in _records("router_examples.txt"):
        z = _floats(r["logits"])
        E = z.shape[0]
        k = int(r["k"])
        idx, w, gap = oracle.route(np.ones((1, 1), np.float32), z[:, None],
                                   _floats(r["bias"]), k)
        np.testing.assert_array_equal(idx[0], [int(v) for v in r["idx"].split()])
        np.testing.assert_allclose(w[0], _floats(r["w"]), rtol=0, atol=2e-7)
        assert gap[0] >= 0


def _brute_topk(x, wr, b, k):
    """Reference selection with a library sort (lexsort: score desc, index asc)."""
    z = x.astype(np.float64) @ wr.astype(np.float64).T
    s = 1 / (1 + np.exp(-z))
    sel = s + b.astype(np.float64)
    out = []
    for t in range(x.shape[0]):
        order = np.lexsort((np.arange(wr.shape[0]), -sel[t]))
        out.append(order[:k])
    return np.array(out), s


def test_router_matches_library_sort_and_invariants():
    rng = np.random.default_rng(11)
    T, H, E, k = 40, 32, 16, 4
    x = rng.standard_normal((T, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.2).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, E).astype(np.float32)
    idx, w, gap = oracle.route(x, wr, b, k)
    ref, s = _brute_topk(x, wr, b, k)
    np.testing.assert_array_equal(idx, ref)
    # renormalised weights sum to one (f32 rounding of k terms)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1) <= k * 2.0 ** -23)
    # the bias picks, the unbiased scores weigh
    want = np.take_along_axis(s, ref, 1)
    np.testing.assert_allclose(w, want / want.sum(1, keepdims=True), rtol=1e-6)
    # without renormalisation the weights are the raw scores times routed_scale
    _, w2, _ = oracle.route(x, wr, b, k, routed_scale=2.5, norm_topk=False)
    np.testing.assert_allclose(w2, 2.5 * want, rtol=1e-6)
    # gap = sel_(k) - sel_(k+1)
    sel = s + b.astype(np.float64)
    srt = -np.sort(-sel, axis=1)
    np.testing.assert_allclose(gap, srt[:, k - 1] - srt[:, k], rtol=1e-9, atol=1e-12)


def test_router_ties_go_to_lower_index():
    E, k = 8, 3
    idx, w, _ = oracle.route(np.zeros((2, 4), np.float32), np.zeros((E, 4), np.float32),
                             np.array([0, 1, 0, 1, 0, 1, 1, 0], np.float32) * 1e-3, k)
    np.testing.assert_array_equal(idx, [[1, 3, 5]] * 2)
    np.testing.assert_allclose(w, 1 / 3, rtol=1e-7)


# --------------------------------------------------------------------------
# union
# --------------------------------------------------------------------------

def test_union_matches_stable_sort():
    rng = np.random.default_rng(5)
    T, k, E = 37, 4, 16
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, ptok, pslot, uniq, n = oracle.union(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")      # library stable sort by expert
    np.testing.assert_array_equal(ptok, order // k)
    np.testing.assert_array_equal(pslot, order % k)
    np.testing.assert_array_equal(offsets, np.searchsorted(np.sort(flat), np.arange(E + 1)))
    np.testing.assert_array_equal(uniq, np.unique(flat))
    assert n == len(np.unique(flat)) and offsets[-1] == T * k
    assert np.all(np.diff(offsets) >= 0)
    seen = set(zip(ptok.tolist(), pslot.tolist()))
    assert len(seen) == T * k


# --------------------------------------------------------------------------
# layer
# --------------------------------------------------------------------------

def _mats(spec, rows, cols):
    return np.array([[float(v) for v in blk.split()] for blk in spec.split("|")],
                    np.float32).reshape(-1, rows, cols)


def test_layer_hand_example():
    r = _records("layer_example.txt")[0]
    x = _floats(r["x"])[None, :]
    wr = _mats(r["router"], 1, 2)[:, 0, :]
    bias = _floats(r["bias"])
    gate = _mats(r["gate"], 2, 2)
    up = _mats(r["up"], 2, 2)
    down = _mats(r["down"], 2, 2)
    y, idx, w = oracle.layer_forward(x, wr, bias, gate, up, down, k=2, n_shared=1, group=0)
    silu = lambda a: a / (1 + math.exp(-a))
    h0, h2, hs = silu(4.0) * 6, silu(-1.75) * 1.125, silu(3.5) * 1.75
    want = [0.75 * 1.75 * h0 + 0.25 * 3.5 * h2 - 7 * hs,
            0.75 * -0.875 * h0 + 0.25 * 7 * h2 + 0.4375 * hs]
    np.testing.assert_array_equal(idx[0], [0, 2])
    np.testing.assert_allclose(w[0], [0.75, 0.25], atol=3e-7)
    np.testing.assert_allclose(y[0], want, rtol=2e-6)


def _rand_layer(rng, H, I, E, n_shared, scale=0.05):
    n = E + n_shared
    g = (rng.standard_normal((n, I, H)) * scale).astype(np.float32)
    u = (rng.standard_normal((n, I, H)) * scale).astype(np.float32)
    d = (rng.standard_normal((n, H, I)) * scale).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
    b = rng.uniform(-0.01, 0.01, E).astype(np.float32)
    return wr, b, g, u, d


@pytest.mark.parametrize("group", [0, 64])
def test_single_expert_reduces_to_dense_swiglu(group):
    """E = 1, k = 1, no shared expert: the layer is a dense SwiGLU FFN on the
    dequantised weights, computed here with library matmuls."""
    rng = np.random.default_rng(21)
    H, I, T = 128, 64, 5
    wr, b, g, u, d = _rand_layer(rng, H, I, 1, 0)
    x = rng.standard_normal((T, H)).astype(np.float32)
    y, idx, w = oracle.layer_forward(x, wr, b, g, u, d, k=1, n_shared=0, group=group)
    deq = lambda m: oracle.dequantize(*oracle.quantize(m, group), m.shape[1], group).astype(np.float64)
    G, U, D = deq(g[0]), deq(u[0]), deq(d[0])
    a = x.astype(np.float64) @ G.T
    hh = a / (1 + np.exp(-a)) * (x.astype(np.float64) @ U.T)
    np.testing.assert_allclose(y, hh @ D.T, rtol=1e-6, atol=1e-7)
    np.testing.assert_array_equal(w, 1.0)


def test_zero_input_gives_zero_output():
    rng = np.random.default_rng(2)
    wr, b, g, u, d = _rand_layer(rng, 64, 64, 8, 1)
    y, idx, _ = oracle.layer_forward(np.zeros((3, 64), np.float32), wr, b, g, u, d,
                                     k=2, n_shared=1, group=64)
    np.testing.assert_array_equal(y, 0.0)
    # with equal scores the bias alone decides the selection
    np.testing.assert_array_equal(np.sort(idx[0]), np.sort(np.argsort(-b)[:2]))


def test_expert_permutation_equivariance_and_token_independence():
    rng = np.random.default_rng(4)
    H, I, E, k, T = 64, 64, 8, 3, 6
    wr, b, g, u, d = _rand_layer(rng, H, I, E, 1)
    x = rng.standard_normal((T, H)).astype(np.float32)
    y, idx, w = oracle.layer_forward(x, wr, b, g, u, d, k=k, n_shared=1, group=0)
    perm = rng.permutation(E)
    full = np.concatenate([perm, [E]])
    y2, idx2, _ = oracle.layer_forward(x, wr[perm], b[perm], g[full], u[full], d[full],
                                       k=k, n_shared=1, group=0)
    np.testing.assert_allclose(y2, y, rtol=1e-6, atol=1e-7)
    np.testing.assert_array_equal(np.sort(perm[idx2], 1), np.sort(idx, 1))
    # each token's output depends only on that token
    y3, _, _ = oracle.layer_forward(x[2:3], wr, b, g, u, d, k=k, n_shared=1, group=0)
    np.testing.assert_array_equal(y3[0], y[2])


def test_token_forward_rows_subset_matches_full():
    rng = np.random.default_rng(9)
    H, I = 64, 32
    mats = [tuple((rng.standard_normal(s) * 0.1).astype(np.float32)
                  for s in ((I, H), (I, H), (H, I))) for _ in range(3)]
    x = rng.standard_normal(H).astype(np.float32)
    w = np.array([0.6, 0.4], np.float32)
    full = oracle.token_forward(x, w, mats, n_shared=1)
    rows = np.array([63, 0, 17], np.int32)
    np.testing.assert_array_equal(oracle.token_forward(x, w, mats, 1, rows=rows), full[rows])


def test_rmsnorm_closed_form():
    x = np.full((2, 8), 3.0, np.float32)
    x[1] = -0.5
    out = oracle.rmsnorm(x, 1e-5)
    np.testing.assert_allclose(out[0], 3 / math.sqrt(9 + 1e-5), rtol=1e-7)
    np.testing.assert_allclose(out[1], -0.5 / math.sqrt(0.25 + 1e-5), rtol=1e-7)
    rng = np.random.default_rng(0)
    z = rng.standard_normal((4, 1000)).astype(np.float32)
    o = oracle.rmsnorm(z, 0.0)
    np.testing.assert_allclose((o.astype(np.float64) ** 2).mean(1), 1.0, rtol=1e-6)


# ---------------------------------------------------------------------------
# FP8 (E4M3, 128 x 128 block scales) -> f32, the step before the int4 container
# ---------------------------------------------------------------------------

def test_e4m3_hand_values():
    codes = np.array([[0x00, 0x80, 0x38, 0x40, 0x3C, 0xB8, 0x7E, 0xFE, 0x08, 0x01, 0x07, 0x30]],
                     np.uint8)
    want = [0.0, -0.0, 1.0, 2.0, 1.5, -1.0, 448.0, -448.0, 2.0 ** -6, 2.0 ** -9,
            7 * 2.0 ** -9, 0.5]
    got = oracle.fp8_block_dequant(codes, np.ones((1, 1), np.float32))[0]
    np.testing.assert_array_equal(got, np.array(want, np.float32))
    assert math.copysign(1.0, got[1]) == -1.0                  # the sign of zero is kept
    nan = oracle.fp8_block_dequant(np.array([[0x7F, 0xFF]], np.uint8), np.ones((1, 1), np.float32))
    assert np.isnan(nan).all()                                  # S.1111.111 is NaN


def test_e4m3_every_code_matches_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8).reshape(1, 256)
    ours = oracle.fp8_block_dequant(codes, np.ones((1, 2), np.float32))[0]
    ref = torch.from_numpy(codes[0].copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    finite = ~np.isnan(ref)
    assert finite.sum() == 254
    np.testing.assert_array_equal(ours[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.isnan(ours[~finite]).all()


def test_fp8_block_scales_cover_ragged_blocks():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    R, K = 300, 260                                  # 3 x 3 blocks, the last ones ragged
    codes = rng.integers(0, 256, (R, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C             # finite codes only
    bs = rng.uniform(1e-4, 1e-2, (3, 3)).astype(np.float32)
    got = oracle.fp8_block_dequant(codes, bs)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    scale = np.repeat(np.repeat(bs, 128, 0), 128, 1)[:R, :K]
    np.testing.assert_array_equal(got.view(np.uint32), (vals * scale).view(np.uint32))
    # the block edges: row 127 uses block row 0, row 128 block row 1
    assert got[127, 0] == np.float32(vals[127, 0] * bs[0, 0])
    assert got[128, 259] == np.float32(vals[128, 259] * bs[1, 2])


# ---------------------------------------------------------------------------
# adaptive expert top-p (a NEXT row: oracle first)
# ---------------------------------------------------------------------------

def test_topp_hand_examples():
    # dyadic weights: every sum below is exact, so p on a boundary is kept exactly
    w = np.array([[0.5, 0.375, 0.125]], np.float32)
    idx = np.array([[4, 2, 9]], np.int32)
    for p, want in [(0.7, [1, 1, 0]), (0.5, [1, 0, 0]), (0.9, [1, 1, 1]), (1.0, [1, 1, 1]),
                    (0.875, [1, 1, 0]), (0.0, [1, 0, 0])]:   # at least one pick is kept
        keep, n = oracle.topp_keep(w, idx, p)
        assert keep[0].tolist() == want, (p, keep)
        assert n[0] == sum(want)
    # the order is by weight, not by pick position (the bias changes the selection)
    keep, _ = oracle.topp_keep(np.array([[0.125, 0.5, 0.375]], np.float32),
                               np.array([[1, 2, 3]], np.int32), 0.7)
    assert keep[0].tolist() == [0, 1, 1]
    # equal weights go to the lower expert index
    keep, _ = oracle.topp_keep(np.full((1, 4), 0.25, np.float32),
                               np.array([[7, 3, 9, 1]], np.int32), 0.5)
    assert keep[0].tolist() == [0, 1, 0, 1]
    # unnormalised weights: the mass is of the renormalised ones (0.5, 0.25, 0.25)
    keep, _ = oracle.topp_keep(np.array([[1.0, 0.5, 0.5]], np.float32),
                               np.array([[0, 2, 1]], np.int32), 0.75)
    assert keep[0].tolist() == [1, 0, 1]


def test_topp_is_the_smallest_set_reaching_p_by_brute_force():
    import itertools
    rng = np.random.default_rng(9)
    k = 6
    for trial in range(300):
        w = rng.dirichlet(np.ones(k)).astype(np.float32)
        idx = rng.permutation(64)[:k].astype(np.int32)
        p = float(rng.uniform(0.05, 1.0))
        keep, n = oracle.topp_keep(w[None], idx[None], p)
        wn = w.astype(np.float64) / w.astype(np.float64).sum()
        kept = keep[0].astype(bool)
        # no smaller subset reaches p, and the kept one does (or is everything)
        best = min((r for r in range(1, k + 1)
                    if any(wn[list(c)].sum() >= p for c in itertools.combinations(range(k), r))),
                   default=k)
        assert n[0] == best, (w, p, keep)
        assert wn[kept].sum() >= p or n[0] == k
        # the kept picks are the largest weights
        assert wn[kept].min() >= wn[~kept].max(initial=-1.0)


# ---------------------------------------------------------------------------
# 8-bit variant of the container (a NEXT row: oracle first)
# ---------------------------------------------------------------------------

def test_quant8_hand_row_half_to_even():
    # max 127/128 gives s = 1/128 exactly; w/s lands on halves: 2.5 -> 2, 3.5 -> 4
    row = np.array([[127 / 128, 2.5 / 128, 3.5 / 128, -0.5 / 128, -1.5 / 128, 0.0]], np.float32)
    codes, scales = oracle.quantize8(row, 0)
    assert codes[0].tolist() == [127, 2, 4, 0, -2, 0]
    assert scales[0, 0] == np.float32(1 / 128)
    z, zs = oracle.quantize8(np.zeros((1, 64), np.float32), 64)      # zero group: s = 0, q = 0
    assert not z.any() and zs[0, 0] == 0.0


@pytest.mark.parametrize("group", [0, 64])
def test_quant8_roundtrip_and_error_bound(group):
    rng = np.random.default_rng(21 + group)
    R, K = 16, 256
    gs = K if group == 0 else group
    # codes with +-127 in every group and a power-of-two scale: w = q s is a fixed point
    q = rng.integers(-127, 128, (R, K))
    q[:, ::gs] = 127 * rng.choice([-1, 1], (R, K // gs))
    s = (2.0 ** -rng.integers(4, 12, (R, K // gs))).astype(np.float32)
    w = (q * np.repeat(s, gs, 1)).astype(np.float32)
    codes, scales = oracle.quantize8(w, group)
    np.testing.assert_array_equal(codes, q)
    np.testing.assert_array_equal(scales, s)
    np.testing.assert_array_equal(oracle.dequantize8(codes, scales, group), w)
    # random weights: error within half a step, every code in range
    w2 = (rng.standard_normal((R, K)) * 0.02).astype(np.float32)
    c2, s2 = oracle.quantize8(w2, group)
    err = np.abs(oracle.dequantize8(c2, s2, group) - w2)
    assert (err <= np.repeat(s2, gs, 1) / 2 * (1 + 1e-6)).all()
    assert np.abs(c2).max() == 127 and c2.min() >= -127


def test_quant8_groups_reduce_to_per_row_and_reject_bad_shapes():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
    w[:, 0] = 0.1                       # both 64-column groups share the row maximum
    w[:, 64] = -0.1
    c0, s0 = oracle.quantize8(w, 0)
    c64, s64 = oracle.quantize8(w, 64)
    np.testing.assert_array_equal(c0, c64)
    np.testing.assert_array_equal(np.repeat(s0, 2, 1), s64)
    with pytest.raises(RuntimeError):
        oracle.quantize8(np.zeros((2, 96), np.float32), 64)          # 96 not a multiple of 64
    with pytest.raises(RuntimeError):
        oracle.quantize8(np.zeros((2, 64), np.float32), 32)          # group 32 not supported


# ---------------------------------------------------------------------------
# input recipe: the Zipf-skewed prefill router
# ---------------------------------------------------------------------------

def test_prefill_zipf_bias_gives_the_stated_load():
    """The stored bias amplitude routes the prefill workload's own seeded tokens
    so that the busiest expert takes about 100 of the 512 x 8 picks (+-5); the
    least popular ones take a handful (5 with this seed)."""
    import synth
    wl = synth.GLM_PREFILL
    wr, b = synth.router(wl, 0)
    x = synth.tokens(wl, wl.T).numpy()
    idx, _, _ = oracle.route(x, wr.numpy(), b.numpy(), wl.k)
    load = np.bincount(idx.reshape(-1), minlength=wl.E)
    assert 95 <= load.max() <= 105, load.max()
    assert load.min() <= 8
    assert load.sum() == wl.T * wl.k
