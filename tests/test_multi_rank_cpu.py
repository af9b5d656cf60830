"""The multi-GPU bench path on CPU: two `gloo` ranks run bench.py's host-side plumbing
(barrier, max-over-ranks device time, whole-job weak-scaling value, rank-0-only reference
arm). The layer itself shards by tokens into independent replicas, so these are the only
cross-rank steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks(my_ms, world)
        value = bench.weak_scaling_value(4096, world, 20, slowest)
        # the reference arm: only rank 0 works; the others return at once without output
        ran = None
        if rank != 0:
            class A:  # minimal stand-in for parsed arguments (never used past the rank check)
                steps = warmup = gpus = cpu_tokens = 1
                workload = "mixtral_bf16"
            ran = bench.run_reference(A(), rank, world)
        q.put((rank, slowest, value, ran))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, slowest, value, ran in res:
        assert slowest == 15.0  # both ranks see the slowest rank's time
        assert value == pytest.approx(4096 * 2 * 20 / 0.015)
    assert res[1][3] is None


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100, 1, 10, 1000.0) == pytest.approx(1000.0)
    assert not dist.is_initialized()
