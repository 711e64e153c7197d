"""Expert parallelism for the routed MoE layer: one process per GPU, each holding
a contiguous range of the routed experts (rank 0 also the shared experts).

Every rank runs the replicated router and computes, through
coli_moe_layer_set_partition, only the picks whose expert it holds, giving a
partial y; one all-reduce (sum) of the [T, H] f32 partial outputs over the
process group then gives every rank the layer's output.  This module holds the
host logic only (which rank owns which experts, the collective); the layer's
arithmetic runs in libcolimoe.  The pages this layer follows describe its
engine running with all experts resident on six GPUs but give no split; a
contiguous, balanced split by expert index is the plainest one.
"""
from __future__ import annotations

SHARED_RANK = 0  # the rank that computes the shared experts and adds the residual


def expert_range(E: int, rank: int, world: int) -> tuple[int, int]:
    """Routed experts [lo, hi) of a rank: contiguous, sizes differing by at most one."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside [0, {world})")
    return rank * E // world, (rank + 1) * E // world


def owner(e: int, E: int, world: int) -> int:
    """The rank holding routed expert e."""
    for r in range(world):
        lo, hi = expert_range(E, r, world)
        if lo <= e < hi:
            return r
    raise ValueError(f"expert {e} outside [0, {E})")


def combine_partials(y, group=None):
    """Sum the ranks' partial outputs in place (one all-reduce of y)."""
    import torch.distributed as dist
    dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


class ExpertParallelLayer:
    """One rank's share of a layer.  make_layer(expert_range, with_shared) must
    return a DeviceLayer holding those experts (device_layer.DeviceLayer with
    expert_range / with_shared)."""

    def __init__(self, make_layer, E: int, rank: int, world: int, group=None):
        self.rank, self.world, self.group = rank, world, group
        self.range = expert_range(E, rank, world)
        self.layer = make_layer(self.range, rank == SHARED_RANK)

    @property
    def handle(self):
        return self.layer.handle

    def partial(self, x, T, y, ws, residual=None, path=0, idx_out=None, w_out=None, stream=None):
        """This rank's partial y (the residual is added on the shared rank only)."""
        from . import coli_moe_forward_ex
        coli_moe_forward_ex(self.layer.handle, x, T, y, ws,
                            residual=residual if self.rank == SHARED_RANK else None,
                            path=path, idx_out=idx_out, w_out=w_out, stream=stream)
        return y

    def forward(self, x, T, y, ws, residual=None, path=0, stream=None):
        """The layer's output on every rank: partial forward, then the all-reduce."""
        self.partial(x, T, y, ws, residual=residual, path=path, stream=stream)
        return combine_partials(y, self.group)

    def close(self):
        self.layer.close()
