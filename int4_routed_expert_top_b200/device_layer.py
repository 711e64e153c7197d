"""Owning holder for one layer's device buffers (torch CUDA tensors) and its
libcolimoe handle.  It allocates memory and calls the library; every byte of the
expert blobs is written by the library (device quantiser or host packer)."""
from __future__ import annotations

import ctypes

import numpy as np

from . import (Desc, coli_moe_expert_bytes, coli_moe_expert_bytes8, coli_moe_layer_create,
               coli_moe_layer_destroy, coli_moe_layer_set_partition, coli_moe_pack_expert,
               coli_moe_pack_expert8, coli_moe_quantize, coli_moe_quantize_expert8_device,
               coli_moe_quantize_expert_device, coli_moe_workspace_size)


class DeviceLayer:
    """Routed int4 MoE layer resident in HBM.

    router_w [E, H] and router_b [E] are f32 tensors (moved to ``device``).
    Expert weights come either as f32 masters through ``expert_masters(e)``
    returning (gate [I, H], up [I, H], down [H, I]) CUDA tensors, quantised on the
    device, or as ready container arrays through ``container(e)`` returning the
    six numpy arrays of coli_moe_pack_expert.
    """

    def __init__(self, H, I, E, k, n_shared, group, router_w, router_b, *,
                 expert_masters=None, container=None, routed_scale=1.0, norm_topk=True,
                 device="cuda", expert_range=None, with_shared=True, bits=4):
        """expert_range=(lo, hi): hold and compute only routed experts lo <= e < hi
        (and the shared experts when with_shared), as one rank of an
        expert-parallel layer (coli_moe_layer_set_partition).  bits=8: 8-bit
        expert codes (quantised by coli_moe_quantize_expert8_device or packed by
        coli_moe_pack_expert8 from the container arrays of coli_moe_quantize8)."""
        import torch
        self.H, self.I, self.E, self.k = H, I, E, k
        self.n_shared, self.group = n_shared, group
        self.routed_scale, self.norm_topk = routed_scale, norm_topk
        self.bits = bits
        self.blob_bytes = (coli_moe_expert_bytes8 if bits == 8 else coli_moe_expert_bytes)(H, I, group)
        lo, hi = expert_range if expert_range is not None else (0, E)
        self.expert_range = (lo, hi)
        self.with_shared = with_shared or expert_range is None
        ids = list(range(lo, hi)) + (list(range(E, E + n_shared)) if self.with_shared else [])
        self.expert_ids = ids
        self.router_w = router_w.to(device=device, dtype=torch.float32).contiguous()
        self.router_b = router_b.to(device=device, dtype=torch.float32).contiguous()
        self.experts = torch.empty((max(len(ids), 1), self.blob_bytes), dtype=torch.uint8,
                                   device=device)
        for slot, e in enumerate(ids):
            if expert_masters is not None:
                g, u, d = expert_masters(e)
                quant = coli_moe_quantize_expert8_device if bits == 8 else coli_moe_quantize_expert_device
                quant(H, I, group, g.contiguous(), u.contiguous(), d.contiguous(),
                      self.experts[slot])
            else:
                pack = coli_moe_pack_expert8 if bits == 8 else coli_moe_pack_expert
                blob = pack(H, I, group, *container(e))
                self.experts[slot].copy_(torch.from_numpy(blob))
        self.desc = Desc(H, I, E, k, n_shared, group, routed_scale, int(norm_topk),
                         self.router_w.data_ptr(), self.router_b.data_ptr(),
                         self.experts.data_ptr(), bits)
        self.handle = coli_moe_layer_create(self.desc)
        if expert_range is not None:
            coli_moe_layer_set_partition(self.handle, lo, hi, self.with_shared, self.experts)

    def workspace_bytes(self, T: int) -> int:
        return coli_moe_workspace_size(self.handle, T)

    def workspace(self, T: int):
        import torch
        return torch.empty((self.workspace_bytes(T),), dtype=torch.uint8,
                           device=self.experts.device)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            coli_moe_layer_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def container_from_masters(gate: np.ndarray, up: np.ndarray, down: np.ndarray, group: int):
    """Host quantisation of one expert into the six container arrays."""
    gc, gs = coli_moe_quantize(gate, group)
    uc, us = coli_moe_quantize(up, group)
    dc, ds = coli_moe_quantize(down, group)
    return gc, gs, uc, us, dc, ds
