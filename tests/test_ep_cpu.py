"""Expert parallelism, host side, without a GPU: the expert ranges of the ranks
partition the routed experts, and with two gloo ranks the all-reduce of the
ranks' partial outputs (each computed here by the oracle over the picks of its
own experts, the shared expert on rank 0 only) gives the whole layer's output.
The oracle stands in for the rank's kernels; the collective and the
partitioning are the package's own (int4_routed_expert_top_b200.ep)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from int4_routed_expert_top_b200 import ep


@pytest.mark.parametrize("E,world", [(256, 1), (256, 2), (256, 4), (256, 6), (256, 8),
                                     (16, 3), (7, 7), (5, 8)])
def test_expert_ranges_partition_the_experts(E, world):
    ranges = [ep.expert_range(E, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    for (a, b), (c, d) in zip(ranges, ranges[1:]):
        assert b == c                                   # contiguous, disjoint
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1                 # balanced
    for e in range(E):
        r = ep.owner(e, E, world)
        lo, hi = ranges[r]
        assert lo <= e < hi


def _oracle_partial(rank, world, seed):
    import oracle
    import synth
    import dataclasses
    from tests.workloads import OracleExperts
    wl = dataclasses.replace(synth.TINY, T=5, group=64, seed=seed)
    wr, b = synth.router(wl)
    x = synth.tokens(wl, wl.T).numpy()
    idx, w, _ = oracle.route(x, wr.numpy(), b.numpy(), wl.k)
    experts = OracleExperts(wl, device="cpu")
    lo, hi = ep.expert_range(wl.E, rank, world)
    with_shared = rank == ep.SHARED_RANK
    y = np.zeros((wl.T, wl.H), np.float32)
    full = np.zeros((wl.T, wl.H), np.float32)
    for t in range(wl.T):
        wt = np.where((idx[t] >= lo) & (idx[t] < hi), w[t], 0.0).astype(np.float32)
        ex = [experts(int(e)) for e in idx[t]]
        sh = [experts(wl.E + s) for s in range(wl.n_shared)]
        y[t] = oracle.token_forward(x[t], wt, ex + (sh if with_shared else []),
                                    wl.n_shared if with_shared else 0)
        full[t] = oracle.token_forward(x[t], w[t], ex + sh, wl.n_shared)
    return y, full


def _worker(rank, world, port, seed, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        y, full = _oracle_partial(rank, world, seed)
        yt = torch.from_numpy(y)
        ep.combine_partials(yt)
        q.put((rank, float(np.abs(yt.numpy() - full).max() / np.abs(full).max())))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_partial_outputs_all_reduce_to_the_layer():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, 77, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    errs = dict(q.get(timeout=10) for _ in range(world))
    assert max(errs.values()) <= 1e-6, errs
