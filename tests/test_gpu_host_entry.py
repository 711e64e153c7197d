"""The host-buffer entry points (x and y in page-locked host memory) give the
same bytes as the device-buffer calls they wrap, directly and when captured
into a CUDA graph, on every expert path."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
import int4_routed_expert_top_b200 as cm
from tests.workloads import build_layer

pytestmark = pytest.mark.gpu

PATHS = {"gemv": cm.COLI_PATH_GEMV, "fused": cm.COLI_PATH_FUSED, "gemm": cm.COLI_PATH_GEMM,
         "auto": cm.COLI_PATH_AUTO}


def device_forward(L, xd, T, path):
    y = torch.empty((T, L.H), dtype=torch.float32, device="cuda")
    cm.coli_moe_forward_ex(L.handle, xd, T, y, L.workspace(T), path=path)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def host_ws(L, T):
    return torch.empty((cm.coli_moe_host_workspace_size(L.handle, T),), dtype=torch.uint8,
                       device="cuda")


@pytest.mark.parametrize("xdt", ["f32", "bf16"])
@pytest.mark.parametrize("path,T", [("gemv", 3), ("fused", 1), ("fused", 5), ("gemm", 24),
                                    ("auto", 2)])
def test_forward_host_equals_device(path, T, xdt):
    wl = dataclasses.replace(synth.TINY, group=64)
    L = build_layer(wl)
    x = torch.randn((T, wl.H))
    if xdt == "bf16":
        x = x.to(torch.bfloat16)
    xh = x.pin_memory()
    yh = torch.empty((T, wl.H), dtype=torch.float32).pin_memory()
    cm.coli_moe_forward_host(L.handle, xh, T, yh, host_ws(L, T), path=PATHS[path])
    torch.cuda.synchronize()
    ref = device_forward(L, x.cuda(), T, PATHS[path])
    np.testing.assert_array_equal(yh.numpy().view(np.uint32), ref.view(np.uint32))


def test_forward_host_in_a_graph_reads_the_current_host_tokens():
    wl = dataclasses.replace(synth.TINY, group=0)
    L = build_layer(wl)
    T = 1
    xh = torch.randn((T, wl.H)).pin_memory()
    yh = torch.empty((T, wl.H), dtype=torch.float32).pin_memory()
    ws = host_ws(L, T)
    cm.coli_moe_forward_host(L.handle, xh, T, yh, ws)      # warm, outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cm.coli_moe_forward_host(L.handle, xh, T, yh, ws)
    for _ in range(3):                                      # new tokens each replay
        x = torch.randn((T, wl.H))
        xh.copy_(x)
        g.replay()
        torch.cuda.synchronize()
        ref = device_forward(L, x.cuda(), T, cm.COLI_PATH_AUTO)
        np.testing.assert_array_equal(yh.numpy().view(np.uint32), ref.view(np.uint32))


def test_stack_forward_host_equals_device():
    wl = dataclasses.replace(synth.TINY, group=64)
    layers = [build_layer(wl, layer=l) for l in range(3)]
    hs = [L.handle for L in layers]
    T = 4
    x = torch.randn((T, wl.H))
    xd = x.cuda()
    ws = torch.empty((cm.coli_moe_stack_workspace_size(hs, T),), dtype=torch.uint8,
                     device="cuda")
    cm.coli_moe_stack_forward(hs, xd, T, 1e-5, ws)
    xh = x.pin_memory()
    yh = torch.empty((T, wl.H), dtype=torch.float32).pin_memory()
    wsh = torch.empty((cm.coli_moe_stack_host_workspace_size(hs, T),), dtype=torch.uint8,
                      device="cuda")
    cm.coli_moe_stack_forward_host(hs, xh, yh, T, 1e-5, wsh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(yh.numpy().view(np.uint32), xd.cpu().numpy().view(np.uint32))
    np.testing.assert_array_equal(xh.numpy(), x.numpy())   # the host input is left as it was


def test_forward_host_rejects_a_short_workspace():
    wl = synth.TINY
    L = build_layer(wl)
    T = 2
    xh = torch.randn((T, wl.H)).pin_memory()
    yh = torch.empty((T, wl.H)).pin_memory()
    short = L.workspace(T)          # the device forward's size: no room for the staging
    with pytest.raises(cm.ColiError) as ei:
        cm.coli_moe_forward_host(L.handle, xh, T, yh, short)
    assert ei.value.code == -5      # COLI_E_WORKSPACE


@pytest.mark.parametrize("path", ["fused", "gemm"])
def test_forward_host_pageable_buffers_use_plain_copies(path):
    """Unpinned host memory is not mapped into the device: the call copies
    through cudaMemcpyAsync instead, with the same result."""
    wl = dataclasses.replace(synth.TINY, group=64)
    L = build_layer(wl)
    T = 1 if path == "fused" else 24
    x = torch.randn((T, wl.H))
    y = torch.empty((T, wl.H), dtype=torch.float32)
    assert not x.is_pinned() and not y.is_pinned()
    cm.coli_moe_forward_host(L.handle, x, T, y, host_ws(L, T), path=PATHS[path])
    torch.cuda.synchronize()
    ref = device_forward(L, x.cuda(), T, PATHS[path])
    np.testing.assert_array_equal(y.numpy().view(np.uint32), ref.view(np.uint32))


def test_forward_host_misaligned_output_is_staged():
    """y_host 4 bytes past a 16-byte boundary: the tensor-core path's 16-byte
    stores cannot target it, so y is staged on the device and copied back."""
    wl = dataclasses.replace(synth.TINY, group=64)
    L = build_layer(wl)
    T = 24
    x = torch.randn((T, wl.H)).pin_memory()
    big = torch.zeros((T * wl.H + 4,), dtype=torch.float32).pin_memory()
    y = big[1:1 + T * wl.H].view(T, wl.H)
    assert y.data_ptr() % 16 == 4
    cm.coli_moe_forward_host(L.handle, x, T, y, host_ws(L, T), path=cm.COLI_PATH_GEMM)
    torch.cuda.synchronize()
    ref = device_forward(L, x.cuda(), T, cm.COLI_PATH_GEMM)
    np.testing.assert_array_equal(y.numpy().view(np.uint32), ref.view(np.uint32))
    assert big[0].item() == 0.0 and big[-3:].abs().sum().item() == 0.0   # nothing outside y
