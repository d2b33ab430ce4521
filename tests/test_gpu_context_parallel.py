"""Context-parallel decode on one GPU: R ranks are emulated as R page-table views of one
packed cache (rank r sees only its page-aligned slice of every sequence, at local
positions 0..n-1).  Each view's partial state is computed by its own launch -- no kernel
waits on another -- and the merged output is compared with the oracle's decode over the
whole context."""
import socket

import numpy as np
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl
from rotated_bit_kv_isoquant_b200.context_parallel import ContextParallelDecoder, slice_of
from _gpu_util import Run, check_attention, log_record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _rank_views(run: Run, lens, R):
    """Per emulated rank: a view of its slice of the cache and its local lengths."""
    return [slice_of(run.cache, run.layout.page_table, lens, R, r) for r in range(R)]


def _cp_decode(run: Run, Q, lens, R, order=None):
    cfg = run.cfg
    views = _rank_views(run, lens, R)
    states = torch.empty((R, Q.shape[0], Q.shape[1], cfg.d + 4), dtype=torch.float32,
                         device="cuda")
    for r, (view, local) in enumerate(views):
        mx = max(local)
        nb = iq.isoq_decode_workspace_bytes(Q.shape[0], Q.shape[1], cfg.n_kv_heads, cfg.d, mx)
        ws = torch.empty((max(nb, 16),), dtype=torch.uint8, device="cuda")
        sl = torch.tensor(local, dtype=torch.int32, device="cuda")
        iq.isoq_decode_partial_state(run.params, view, Q, sl, mx, states[r], cfg.scale, ws)
    if order is not None:
        states = states[list(order)].contiguous()
    out = torch.empty((Q.shape[0], Q.shape[1], cfg.d), dtype=torch.float32, device="cuda")
    iq.isoq_decode_merge_states(run.params, states, out)
    torch.cuda.synchronize()
    return out, states


@pytest.fixture(scope="module")
def run2():
    cfg = wl.small_variant(wl.workload(2), length=4000)
    r = Run(cfg)
    r.prefill()
    return r


@pytest.fixture(scope="module")
def run4():
    cfg = wl.small_variant(wl.workload(4), n_seqs=5, len_range=(0, 900))
    r = Run(cfg)
    r.prefill()
    r.append()
    return r


@pytest.mark.parametrize("R", [2, 3, 4, 8])
def test_cp_matches_oracle_single_long_sequence(oracle, run2, R):
    Q = wl.queries(run2.cfg, device="cuda")
    lens = run2.cfg.decode_lens()
    out, _ = _cp_decode(run2, Q, lens, R)
    stats = check_attention(oracle, run2, Q, out, lens)
    log_record({"case": f"cp_ctx4000_R{R}", **stats})


def test_cp_one_rank_is_the_plain_decode_bitwise(run2):
    Q = wl.queries(run2.cfg, device="cuda")
    lens = run2.cfg.decode_lens()
    out, _ = _cp_decode(run2, Q, lens, 1)
    _, ref = run2.decode(Q=Q, lens=lens)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_cp_batched_ragged_shuffled_pages(oracle, run4):
    Q = wl.queries(run4.cfg, device="cuda")
    lens = list(run4.cfg.decode_lens())
    lens[1] = 0                      # an empty context: every slice is empty
    lens[2] = min(lens[2], 37)       # shorter than one page: one rank holds it all
    out, states = _cp_decode(run4, Q, lens, 3)
    assert torch.all(states[:, 1, :, run4.cfg.d] == float("-inf"))
    assert torch.all(out[1] == 0)
    stats = check_attention(oracle, run4, Q, out, lens)
    log_record({"case": "cp_batched_R3", **stats})


def test_cp_merge_order_does_not_matter(run2):
    Q = wl.queries(run2.cfg, device="cuda")
    lens = run2.cfg.decode_lens()
    a, _ = _cp_decode(run2, Q, lens, 4)
    b, _ = _cp_decode(run2, Q, lens, 4, order=(3, 1, 0, 2))
    rel = ((a - b).norm() / a.norm()).item()
    assert rel < 1e-6


def test_cp_merge_rejects_bad_arguments(run2):
    out = torch.empty((1, run2.cfg.n_q_heads, run2.cfg.d), device="cuda")
    lib = iq.raw_lib()
    rc = lib.isoq_decode_merge_states(run2.params.handle, out.data_ptr(), 0, 1,
                                      run2.cfg.n_q_heads, out.data_ptr(), None)
    assert rc == iq.ISOQ_E_ARG
    rc = lib.isoq_decode_merge_states(run2.params.handle, out.data_ptr(), 1, 1,
                                      run2.cfg.n_q_heads + 1, out.data_ptr(), None)
    assert rc == iq.ISOQ_E_GQA


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_cp_decoder_over_a_one_rank_nccl_group(oracle, run2):
    """The decoder class end to end, its all-gather on NCCL (a group of one GPU)."""
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        Q = wl.queries(run2.cfg, device="cuda")
        lens = run2.cfg.decode_lens()
        dec = ContextParallelDecoder(run2.params, run2.cache, Q.shape[0], Q.shape[1], max(lens))
        out = torch.empty((Q.shape[0], Q.shape[1], run2.cfg.d), dtype=torch.float32,
                          device="cuda")
        dec(Q, torch.tensor(lens, dtype=torch.int32, device="cuda"), out, run2.cfg.scale)
        torch.cuda.synchronize()
        check_attention(oracle, run2, Q, out, lens)
    finally:
        dist.destroy_process_group()


def test_cp_decoder_on_a_side_stream(oracle, run2):
    """The decoder given a stream other than the current one: the partial state, the
    all-gather (NCCL, a group of one GPU) and the merge all run in order on that stream,
    and the result equals the one on the current stream bitwise."""
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        Q = wl.queries(run2.cfg, device="cuda")
        lens = run2.cfg.decode_lens()
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        dec = ContextParallelDecoder(run2.params, run2.cache, Q.shape[0], Q.shape[1], max(lens))
        ref = torch.empty((Q.shape[0], Q.shape[1], run2.cfg.d), dtype=torch.float32,
                          device="cuda")
        dec(Q, sl, ref, run2.cfg.scale)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        out = torch.full_like(ref, float("nan"))
        dec.state.fill_(float("nan"))
        junk = torch.empty((1 << 26,), device="cuda")
        side.wait_stream(torch.cuda.current_stream())
        # a long kernel on the side stream first, so a merge that ran ahead of the
        # partial state or the gather would read stale data
        with torch.cuda.stream(side):
            junk.normal_()
        dec(Q, sl, out, run2.cfg.scale, stream=side)
        side.synchronize()
        assert torch.equal(out, ref)
        check_attention(oracle, run2, Q, out, lens)
    finally:
        dist.destroy_process_group()
