"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun would start them.
Each rank reports its own timing; the job's number must use the slowest rank (max over
ranks) and count every rank's work (weak scaling)."""
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


def _rank_main(rank, world, port, local_ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rank_env = bench._dist_env()
        mx = bench.max_over_ranks(local_ms[rank], world, "cpu")
        rate = bench.weak_scaling_rate(1000.0, 4, world, mx)
        dist.barrier()
        q.put((rank, rank_env, mx, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_weak_scaling_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    local_ms = [3.0, 5.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, (r, w, lr), mx, rate in got:
        assert (r, w, lr) == (rank, world, rank)
        assert mx == 5.0                                  # the slowest rank's time
        assert rate == pytest.approx(1000.0 * 4 * world / 5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.weak_scaling_rate(10.0, 3, 1, 2.0) == pytest.approx(15000.0)
