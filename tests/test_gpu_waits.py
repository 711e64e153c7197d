"""The fused kernel's bounded waits run out without hanging the GPU: with the
test option of coli_moe_layer_set_wait_test, CTA 0's producer never issues one
ring stage, the consumer warps' wait on it gives up after a short limit, the
kernel and the combine return, coli_moe_status reports COLI_E_TIMEOUT, and the
next call on the same workspace (option cleared) is correct and bit-identical
to a call that never saw the option."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import (OracleExperts, build_layer, gap_resampled_tokens, oracle_tokens,
                             rel_err)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,group", [(1, 0), (4, 64), (12, 64)])
def test_wait_gives_up_and_the_next_call_is_correct(T, group):
    wl = dataclasses.replace(synth.TINY, T=T, group=group)
    wr, b = synth.router(wl)
    x, idx_ref, w_ref, _ = gap_resampled_tokens(wl, T, wr, b)
    y_ref = oracle_tokens(wl, OracleExperts(wl), x.numpy(), idx_ref, w_ref)
    L = build_layer(wl, router=(wr, b))
    ws = L.workspace(T)
    xd = x.cuda()
    y = torch.empty((T, wl.H), dtype=torch.float32, device="cuda")
    cm.coli_moe_forward_ex(L.handle, xd, T, y, ws, path=cm.COLI_PATH_FUSED)
    torch.cuda.synchronize()
    y_clean = y.cpu().numpy().copy()
    assert cm.coli_moe_status(L.handle, T, ws) == 0

    cm.coli_moe_layer_set_wait_test(L.handle, 0)
    cm.coli_moe_forward_ex(L.handle, xd, T, y, ws, path=cm.COLI_PATH_FUSED)
    with pytest.raises(cm.ColiError) as e:
        cm.coli_moe_status(L.handle, T, ws)
    assert e.value.code == -6                                  # COLI_E_TIMEOUT

    cm.coli_moe_layer_set_wait_test(L.handle, -1)
    y.fill_(float("nan"))
    cm.coli_moe_forward_ex(L.handle, xd, T, y, ws, path=cm.COLI_PATH_FUSED)
    torch.cuda.synchronize()
    assert cm.coli_moe_status(L.handle, T, ws) == 0
    out = y.cpu().numpy()
    np.testing.assert_array_equal(out.view(np.uint32), y_clean.view(np.uint32))
    assert rel_err(out, y_ref) <= 2e-3
    L.close()
