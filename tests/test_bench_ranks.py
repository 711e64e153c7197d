"""bench.py with several ranks (one replica per GPU under torchrun): the job's
time is the largest over the ranks and its throughput counts every rank's
tokens; the reference arm runs on rank 0 alone.  Host logic only, checked with
two gloo ranks on the CPU."""
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = [12.5, 20.0][rank]                 # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_tokens_per_s(7, world, job_ms)
        queue.put((rank, job_ms, value))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_job_time_is_the_slowest_rank_and_value_counts_every_rank():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, job_ms, value in results:
        assert job_ms == 20.0
        assert value == pytest.approx(7 * 2 / 20e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.job_tokens_per_s(4, 1, 2.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, timeout=300)
    assert r.returncode == 0, r.stderr.decode()[-500:]
    assert r.stdout.strip() == b""


def test_profiled_traffic_only_while_the_kernel_source_matches(tmp_path):
    """The roofline's traffic comes from an ncu summary only while the kernel
    source still has the hash that summary names."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = "int4_routed_expert_top_b200/csrc/fused.cuh"
    digest = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
    (tmp_path / "p.md").write_text(
        f"source sha256 prefix {digest[:16]}\n\n| metric | value |\n|---|---|\n"
        "| traffic_bytes_per_launch | 173990000 |\n")
    t = bench.profiled_traffic(src, "p.md", str(tmp_path))
    assert t == 173990000.0
    # another source file has another hash: no traffic
    assert bench.profiled_traffic("int4_routed_expert_top_b200/csrc/gemm.cuh", "p.md",
                                  str(tmp_path)) is None
    assert bench.profiled_traffic(src, "no_such_profile.md", str(tmp_path)) is None
