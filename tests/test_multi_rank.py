"""The multi-GPU path of bench.py on CPU: two gloo ranks run the same barrier / max-over-
ranks / whole-job-rate steps that bench.py takes under torchrun (one replica per GPU,
timed on each device, max over ranks)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world)
        rate = bench.whole_job_rate(64 * 100, world, ms)
        # sequence sharding of a 5-sequence batch: every sequence in exactly one shard
        lo, hi = bench.shard_range(5, rank, world)
        seqs = list(range(lo, hi))
        gathered = [None] * world
        dist.all_gather_object(gathered, seqs)
        assert sorted(x for part in gathered for x in part) == list(range(5))
        q.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_rate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [15.0, 15.0]
    # both replicas' tokens over the slowest replica's time
    assert all(abs(g[2] - 2 * 6400 / 0.015) < 1e-6 for g in got)
