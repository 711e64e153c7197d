"""CPU-side checks of libcolimoe: the library loads and exports every symbol the
header declares, the host quantiser is bit-identical to the oracle's, the host
packer follows the documented device layout, and argument errors come back as
status codes.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import int4_routed_expert_top_b200 as cm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_exports_match_header():
    text = open(os.path.join(ROOT, "include", "coli_moe.h")).read()
    declared = set(re.findall(r"^\s*(?:int|const char\*)\s+(coli_moe_\w+)\(", text, re.M))
    assert declared == set(cm.EXPORTS)
    for name in declared:
        assert hasattr(cm.lib, name), name
        assert callable(getattr(cm, name)), name


@pytest.mark.parametrize("group", [0, 64])
def test_host_quantizer_bit_identical_to_oracle(group):
    rng = np.random.default_rng(17)
    w = (rng.standard_normal((96, 384)) * 0.02).astype(np.float32)
    w[3] = 0.0
    w[7, ::5] = 0.0035          # ties at exact multiples of the scale
    p0, s0 = oracle.quantize(w, group)
    p1, s1 = cm.coli_moe_quantize(w, group)
    np.testing.assert_array_equal(p0, p1)
    np.testing.assert_array_equal(s0.view(np.uint32), s1.view(np.uint32))


def test_host_quantizer_golden_rows():
    row = np.array([[3.5, 1.25, -0.75, 0.25]], np.float32)
    p, s = cm.coli_moe_quantize(row, 0)
    assert p.tobytes().hex() == "270e" and s[0, 0] == 0.5


def _unpack_blob(blob, H, I, group):
    """Read a blob back through the layout the header documents."""
    def sec_align(v):
        return (v + 255) // 256 * 256
    mats = [(I, H), (I, H), (H, I)]
    off = 0
    code_off = []
    for R, K in mats:
        code_off.append(off)
        off = sec_align(off + R * K // 2)
    scale_off = []
    for R, K in mats:
        ng = 1 if group == 0 else K // group
        scale_off.append(off)
        off = sec_align(off + R * ng * 4)
    assert off == blob.size
    # word j of unit (t, s, b, l): nibble p at bits 4p.. holds
    #   p: 0 (r1,c0) 1 (r0,c0) 2 (r1,c0+1) 3 (r0,c0+1) 4 (r1,c0+2) 5 (r0,c0+2)
    #      6 (r1,c0+3) 7 (r0,c0+3); r0 = 128t + 16b + l//4, r1 = r0 + 8,
    #   c0 = 64s + 16j + 4(l%4)
    dr = np.array([8, 0, 8, 0, 8, 0, 8, 0])
    dc = np.array([0, 0, 1, 1, 2, 2, 3, 3])
    out = []
    for m, (R, K) in enumerate(mats):
        ng = 1 if group == 0 else K // group
        words = blob[code_off[m]:code_off[m] + R * K // 2].view(np.uint32)
        words = words.reshape(R // 128, K // 64, 8, 32, 4)
        t, s_, b, l, j = np.meshgrid(*[np.arange(n) for n in words.shape], indexing="ij")
        r0 = 128 * t + 16 * b + l // 4
        c0 = 64 * s_ + 16 * j + 4 * (l % 4)
        q = np.zeros((R, K), np.uint8)
        for p in range(8):
            q[r0 + dr[p], c0 + dc[p]] = (words >> (4 * p)) & 15
        codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
        sc = blob[scale_off[m]:scale_off[m] + R * ng * 4].view(np.float32)
        sc = sc.reshape(R // 128, ng, 128).transpose(0, 2, 1).reshape(R, ng)
        out += [codes, sc]
    return out


@pytest.mark.parametrize("group", [0, 64])
def test_pack_expert_follows_documented_layout(group):
    rng = np.random.default_rng(1)
    H, I = 256, 128
    mats = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in ((I, H), (I, H), (H, I))]
    cont = []
    for m in mats:
        cont += list(cm.coli_moe_quantize(m, group))
    blob = cm.coli_moe_pack_expert(H, I, group, *cont)
    assert blob.size == cm.coli_moe_expert_bytes(H, I, group)
    back = _unpack_blob(blob, H, I, group)
    for a, b in zip(cont, back):
        np.testing.assert_array_equal(a, b)


def test_expert_bytes_glm():
    # codes 3 * 6144 * 2048 / 2 plus per-row scales (2048 + 2048 + 6144) * 4
    assert cm.coli_moe_expert_bytes(6144, 2048, 0) == 18874368 + 40960
    # gs64: (2048 * 96 * 2 + 6144 * 32) * 4 scale bytes
    assert cm.coli_moe_expert_bytes(6144, 2048, 64) == 18874368 + 2359296


def test_argument_errors_are_status_codes():
    with pytest.raises(cm.ColiError) as e:
        cm.coli_moe_quantize(np.zeros((2, 3), np.float32), 0)
    assert e.value.code == -1 and "bad shape" in str(e.value)
    with pytest.raises(cm.ColiError):
        cm.coli_moe_expert_bytes(100, 128, 0)           # H not a multiple of 128
    with pytest.raises(cm.ColiError):
        cm.coli_moe_expert_bytes(256, 128, 32)          # unsupported group
    d = cm.Desc(256, 128, 16, 4, 1, 0, 1.0, 1, 0, 0, 0)  # NULL device pointers
    with pytest.raises(cm.ColiError):
        cm.coli_moe_layer_create(d)
    d = cm.Desc(256, 128, 16, 17, 1, 0, 1.0, 1, 16, 16, 16)  # k > E
    with pytest.raises(cm.ColiError):
        cm.coli_moe_layer_create(d)


def test_workspace_size_and_limits_without_gpu():
    # placeholder non-null addresses: layer_create only validates, never touches them
    d = cm.Desc(6144, 2048, 256, 8, 1, 64, 1.0, 1, 256, 256, 256)
    h = cm.coli_moe_layer_create(d)
    try:
        small, big = cm.coli_moe_workspace_size(h, 1), cm.coli_moe_workspace_size(h, 512)
        assert 0 < small < big
        # f32 h and o for every (token, expert) pair dominate the workspace
        assert big >= 512 * 9 * (2048 + 6144) * 4
        with pytest.raises(cm.ColiError):
            cm.coli_moe_workspace_size(h, 0)
        with pytest.raises(cm.ColiError) as e:
            cm.coli_moe_workspace_size(h, 8192)         # union bitmap limit
        assert e.value.code == -4
        # the host-buffer calls add staging for x and y behind the forward's workspace
        hb = cm.coli_moe_host_workspace_size(h, 4)
        assert hb >= cm.coli_moe_workspace_size(h, 4) + 2 * 4 * 6144 * 4
        sb = cm.coli_moe_stack_host_workspace_size([h, h], 4)
        assert sb >= cm.coli_moe_stack_workspace_size([h, h], 4) + 4 * 6144 * 4
        # a workspace that is too small is refused before anything is launched
        ws = np.zeros(16, np.uint8)
        with pytest.raises(cm.ColiError) as e:
            rc = cm.lib.coli_moe_forward(h, 256, 0, 1, 256, ws.ctypes.data, 16, None)
            cm._ok(rc)
        assert e.value.code == -5
    finally:
        cm.coli_moe_layer_destroy(h)


# ---------------------------------------------------------------------------
# 8-bit codes: host quantiser and packer (the expert kernels do not read them yet)
# ---------------------------------------------------------------------------

def _unpack_blob8(blob, H, I, group):
    """Read an 8-bit blob back through the layout the header documents."""
    def sec_align(v):
        return (v + 255) // 256 * 256
    mats = [(I, H), (I, H), (H, I)]
    off, code_off, scale_off = 0, [], []
    for R, K in mats:
        code_off.append(off)
        off = sec_align(off + R * K)
    for R, K in mats:
        ng = 1 if group == 0 else K // group
        scale_off.append(off)
        off = sec_align(off + R * ng * 4)
    assert off == blob.size
    out = []
    for m, (R, K) in enumerate(mats):
        ng = 1 if group == 0 else K // group
        # [T][s][b][lane][h][i][j]: word i of half h, byte j
        raw = blob[code_off[m]:code_off[m] + R * K].view(np.int8)
        raw = raw.reshape(R // 128, K // 64, 8, 32, 2, 4, 4)
        T, s_, b, l, h, i, j = np.meshgrid(*[np.arange(n) for n in raw.shape], indexing="ij")
        r = 128 * T + 16 * b + l // 4 + 8 * (i % 2)          # i = 1, 3: row r0 + 8
        c = 64 * s_ + 32 * h + 4 * (l % 4) + 16 * (i // 2) + j  # i = 2, 3: columns + 16
        q = np.zeros((R, K), np.int8)
        q[r, c] = raw
        sc = blob[scale_off[m]:scale_off[m] + R * ng * 4].view(np.float32)
        sc = sc.reshape(R // 128, ng, 128).transpose(0, 2, 1).reshape(R, ng)
        out += [q, sc]
    return out


@pytest.mark.parametrize("group", [0, 64])
def test_quantize8_bit_identical_to_oracle(group):
    rng = np.random.default_rng(4 + group)
    w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    w[3, 10] = 0.0
    w[5, :] = 0.0                                   # a zero row
    c, s = cm.coli_moe_quantize8(w, group)
    co, so = oracle.quantize8(w, group)
    np.testing.assert_array_equal(c, co)
    np.testing.assert_array_equal(s.view(np.uint32), so.view(np.uint32))
    row = np.array([[127 / 128, 2.5 / 128, 3.5 / 128, -0.5 / 128, -1.5 / 128, 0.0]], np.float32)
    assert cm.coli_moe_quantize8(row, 0)[0][0].tolist() == [127, 2, 4, 0, -2, 0]


@pytest.mark.parametrize("group", [0, 64])
def test_pack_expert8_follows_documented_layout(group):
    rng = np.random.default_rng(2)
    H, I = 256, 128
    mats = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in ((I, H), (I, H), (H, I))]
    cont = []
    for m in mats:
        cont += list(cm.coli_moe_quantize8(m, group))
    blob = cm.coli_moe_pack_expert8(H, I, group, *cont)
    assert blob.size == cm.coli_moe_expert_bytes8(H, I, group)
    back = _unpack_blob8(blob, H, I, group)
    for a, b in zip(cont, back):
        np.testing.assert_array_equal(a, b)


def test_expert_bytes8_glm():
    codes = 3 * 6144 * 2048                       # one byte per weight
    assert cm.coli_moe_expert_bytes8(6144, 2048, 0) == codes + 40960
    assert cm.coli_moe_expert_bytes8(6144, 2048, 64) == codes + 2359296
