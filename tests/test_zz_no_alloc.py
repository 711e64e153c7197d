"""The allocation-free forward (coli_moe_forward_noalloc), for callers that
cannot allocate device memory, against the ordinary forward with a caller
workspace.  Kept in its own file, collected last, so that a run stopping at the
first failure has already run every other test."""
import numpy as np
import pytest
import torch

import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import build_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("group", [0, 64])
def test_noalloc_forward_matches_workspace_forward(group):
    """Same path as the ordinary forward (the fused kernel here), so the same
    bytes, on two calls in a row that share the built-in scratch array; the
    array's error flags read back clear afterwards."""
    import dataclasses
    wl = dataclasses.replace(synth.TINY, group=group, T=5)
    L = build_layer(wl)
    y_ref = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    y = torch.empty_like(y_ref)
    for call in range(2):
        x = synth.tokens(wl, wl.T, step=call).cuda()
        cm.coli_moe_forward(L.handle, x, wl.T, y_ref, L.workspace(wl.T))
        y.fill_(float("nan"))
        cm.coli_moe_forward_noalloc(L.handle, x, wl.T, y)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32),
                                      y_ref.cpu().numpy().view(np.uint32))
        assert cm.coli_moe_status(L.handle, wl.T, None) == 0
    L.close()


def test_noalloc_rejects_too_many_tokens():
    """8192 tokens of the tiny layer: even the GEMV path's workspace prefix (its
    fp16 activation digits alone are T * H * 4 = 8 MiB) exceeds the array."""
    wl = synth.TINY
    L = build_layer(wl)
    T = 8192
    x = torch.zeros((T, wl.H), dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    with pytest.raises(cm.ColiError) as e:
        cm.coli_moe_forward_noalloc(L.handle, x, T, y)
    assert e.value.code == -4 and "scratch" in str(e.value)
    L.close()


def test_noalloc_uses_the_gemv_path_when_the_fused_scratch_does_not_fit():
    """H 4096, I 1024, 16 tokens: the fused path's partial products need more than
    the built-in array, the GEMV path's workspace fits, so the call runs the GEMV
    path and gives exactly its bytes (and the oracle-checked path's values)."""
    import dataclasses
    wl = dataclasses.replace(synth.TINY, H=4096, I=1024, T=16)
    L = build_layer(wl)
    assert cm.coli_moe_workspace_size(L.handle, wl.T) > cm.NOALLOC_SCRATCH_BYTES
    x = synth.tokens(wl, wl.T).cuda()
    y_gemv = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    y_auto = torch.empty_like(y_gemv)
    y = torch.empty_like(y_gemv)
    ws = L.workspace(wl.T)
    cm.coli_moe_forward_ex(L.handle, x, wl.T, y_gemv, ws, path=cm.COLI_PATH_GEMV)
    cm.coli_moe_forward_ex(L.handle, x, wl.T, y_auto, ws, path=cm.COLI_PATH_AUTO)
    for _ in range(2):
        y.fill_(float("nan"))
        cm.coli_moe_forward_noalloc(L.handle, x, wl.T, y)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32),
                                      y_gemv.cpu().numpy().view(np.uint32))
    assert rel_err(y.cpu().numpy(), y_auto.cpu().numpy()) <= 2e-3
    L.close()
