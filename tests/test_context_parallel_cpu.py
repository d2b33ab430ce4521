"""Host logic of the context-parallel decode, on CPU: the page-aligned sharding of a
context over ranks, and the all-gather of the ranks' softmax states over a real process
group (gloo, world size 2 and 3, as torchrun would start the ranks)."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rotated_bit_kv_isoquant_b200.context_parallel import gather_states, shard_tokens


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("seq_len", [0, 1, 63, 64, 65, 1000, 4096, 131072, 131073])
def test_shards_partition_the_context_on_page_boundaries(seq_len, world):
    ranges = [shard_tokens(seq_len, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == seq_len
    for (a0, b0), (a1, b1) in zip(ranges, ranges[1:]):
        assert b0 == a1                       # contiguous, disjoint
    for a, b in ranges:
        assert a <= b
        assert a % 64 == 0 or a == b == seq_len  # a slice starts on a page (or is empty)
    pages = [-(-(b - a) // 64) for a, b in ranges]
    assert max(pages) - min(pages) <= 1       # balanced to one page
    assert sum(b - a for a, b in ranges) == seq_len


def test_shard_rejects_bad_requests():
    for args in [(10, 0, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ValueError):
            shard_tokens(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # a state tensor [n_seqs][n_q_heads][d + 4] whose values name the rank
        st = torch.arange(2 * 3 * 12, dtype=torch.float32).reshape(2, 3, 12) + 1000.0 * rank
        got = gather_states(st)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gather_states_orders_by_rank_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    base = torch.arange(2 * 3 * 12, dtype=torch.float32).reshape(2, 3, 12)
    for rank, got in res:
        assert got.shape == (world, 2, 3, 12)
        for r in range(world):                # every rank sees every rank's state, in order
            assert torch.equal(got[r], base + 1000.0 * r)
