"""GPU parity of 8-bit expert weights (the engine keeps its MTP head at 8 bits:
"解密GLM-5.2-colibri-int4-with-int8-mtp"): the device 8-bit quantiser against the
oracle's quantiser and the host packer byte for byte, dequantised weights bit
for bit, and the fused path's layer outputs against an oracle forward built on
orc_dequantize8 within the fused path's 2e-3."""
import concurrent.futures as cf
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import (OracleExperts, build_layer, gap_resampled_tokens, masters,
                             oracle_tokens, rel_err, same_selection)

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.mark.parametrize("group", [0, 64])
@pytest.mark.parametrize("shape", [(256, 128), (6144, 2048)])
def test_device_quantizer8_matches_host_packer(group, shape):
    H, I = shape
    wl = dataclasses.replace(synth.TINY, H=H, I=I, group=group)
    g, u, d = masters(wl, 0, 5)
    blob = torch.empty(cm.coli_moe_expert_bytes8(H, I, group), dtype=torch.uint8, device="cuda")
    cm.coli_moe_quantize_expert8_device(H, I, group, g, u, d, blob)
    cont = []
    for m in (g, u, d):
        cont += list(oracle.quantize8(m.cpu().numpy(), group))
    host = cm.coli_moe_pack_expert8(H, I, group, *cont)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(blob.cpu().numpy(), host)


@pytest.mark.parametrize("group", [0, 64])
def test_dequant8_bit_exact(group):
    wl = dataclasses.replace(synth.TINY, group=group)
    L = build_layer(wl, bits=8)
    ref = OracleExperts(wl, bits=8)
    for e in (0, 9, wl.E):
        for which in range(3):
            R, K = (wl.I, wl.H) if which < 2 else (wl.H, wl.I)
            out = torch.empty((R, K), dtype=torch.float32, device="cuda")
            cm.coli_moe_dequant_debug(L.handle, e, which, out)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32),
                                          ref(e)[which].view(np.uint32))
    L.close()


def forward(L, x, T, path=cm.COLI_PATH_FUSED):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    cm.coli_moe_forward_ex(L.handle, x, T, y, L.workspace(T), path=path, idx_out=idx)
    torch.cuda.synchronize()
    return y.cpu().numpy(), idx.cpu().numpy()


VARIANTS = {"T1": dict(T=1), "T4": dict(T=4), "T4_gs64": dict(T=4, group=64),
            "T9_gs64": dict(T=9, group=64), "T40": dict(T=40), "no_shared": dict(n_shared=0),
            "three_tiles": dict(H=384, I=256, E=24, k=6, group=64, T=5),
            "bf16_x": dict(x_dtype="bf16", group=64, T=3)}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_layer_parity_int8_small(name):
    wl = dataclasses.replace(synth.TINY, **VARIANTS[name])
    if wl.H % 256:
        pytest.skip("the fused path needs H a multiple of 256")
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, wl.T, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl, bits=8), x.numpy(), idx_ref, w_ref)
    L = build_layer(wl, router=(wr, b), bits=8)
    xd = (x.to(torch.bfloat16) if wl.x_dtype == "bf16" else x).cuda().contiguous()
    y, idx = forward(L, xd, wl.T)
    same_selection(idx, idx_ref)
    err = rel_err(y, y_ref)
    assert err <= TOL, err
    y2, _ = forward(L, xd, wl.T, cm.COLI_PATH_AUTO)      # AUTO takes the fused path
    np.testing.assert_array_equal(y2.view(np.uint32), y.view(np.uint32))
    for path in (cm.COLI_PATH_GEMV, cm.COLI_PATH_GEMM):   # the other paths read 4-bit codes
        with pytest.raises(cm.ColiError) as ei:
            forward(L, xd, wl.T, path)
        assert ei.value.code == -4
    L.close()


@pytest.mark.parametrize("group", [0, 64])
def test_glm_int8_layer(group):
    """GLM-5.2-shaped layer with 8-bit experts (257 resident, ~9.7 GB per-row or
    10.9 GB gs64): one token and a batch of 3, every output against the oracle."""
    wl = dataclasses.replace(synth.GLM_DECODE, group=group, seed=6006 + group)
    L = build_layer(wl, bits=8)
    wr, b = L.router_w.cpu(), L.router_b.cpu()
    experts = OracleExperts(wl, bits=8)
    for T in (1, 3):
        x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, T, wr, b, step=T)
        with cf.ThreadPoolExecutor(16) as ex:
            list(ex.map(experts, sorted({int(e) for e in idx_ref.ravel()} | {wl.E})))
        y, idx = forward(L, x.cuda(), T)
        same_selection(idx, idx_ref)
        y_ref = oracle_tokens(wl, experts, x.numpy(), idx_ref, w_ref)
        err = rel_err(y, y_ref)
        print(f"GLM 8-bit layer group {group}, T={T}: rel err {err:.2e}")
        assert err <= TOL, (T, err)
        experts.cache.clear()
    L.close()
    torch.cuda.empty_cache()
