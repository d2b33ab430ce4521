"""Multi-token (chunked-prefill / speculative-verify) attention on the packed cache against
the fp64 oracle.  Query token i of a chunk of n_q sits at position L - n_q + i and attends
cache positions 0 .. L - n_q + i, so its reference is the oracle's decode of one query
over that prefix of the same packed cache (host copy): each (sequence, i) becomes one
oracle "sequence" whose page-table row is the sequence's and whose length is that prefix."""
import numpy as np
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl
from _gpu_util import ATTN_TOL, Run, log_record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _multi(run: Run, Q, lens, max_len=None):
    cfg = run.cfg
    n_seqs, n_q, hq = Q.shape[0], Q.shape[1], Q.shape[2]
    max_len = max(lens) if max_len is None else max_len
    nb = iq.isoq_multi_token_workspace_bytes(n_seqs, n_q, hq, cfg.n_kv_heads, cfg.d, max_len)
    ws = torch.empty((max(nb, 16),), dtype=torch.uint8, device="cuda")
    out = torch.full((n_seqs, n_q, hq, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    iq.isoq_multi_token_attention(run.params, run.cache, Q, sl, max_len, out, cfg.scale, ws)
    torch.cuda.synchronize()
    return out


def _oracle_multi(oracle, run: Run, Q, lens):
    cfg = run.cfg
    n_seqs, n_q = Q.shape[0], Q.shape[1]
    pt = run.layout.page_table.numpy()
    rows = [(s, i) for s in range(n_seqs) for i in range(n_q)]
    vpt = np.stack([pt[s] for s, _ in rows])
    vlen = [max(0, lens[s] - n_q + i + 1) for s, i in rows]
    q = Q.float().cpu().numpy().astype(np.float64).reshape(n_seqs * n_q, Q.shape[2], cfg.d)
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64,
                                  run.cache.blocks.cpu().numpy(), vpt, vlen, q, cfg.scale)
    return ref.reshape(n_seqs, n_q, Q.shape[2], cfg.d)


def _compare(ref, got):
    got = got.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    r = ref.reshape(-1, ref.shape[-1])
    g = got.reshape(-1, got.shape[-1])
    nr = np.linalg.norm(r, axis=1)
    zero = nr == 0
    assert np.all(np.linalg.norm(g[zero], axis=1) == 0)
    err = np.linalg.norm(g[~zero] - r[~zero], axis=1) / nr[~zero]
    assert err.max() <= ATTN_TOL, f"max rel L2 {err.max()}"
    return {"rows": int(r.shape[0]), "max_rel": float(err.max()), "mean_rel": float(err.mean())}


@pytest.fixture(scope="module")
def run2():
    r = Run(wl.small_variant(wl.workload(2), length=3000))
    r.prefill()
    return r


@pytest.mark.parametrize("n_q", [1, 2, 7, 16, 64])
def test_multi_token_chunk_matches_oracle(oracle, run2, n_q):
    Q = wl.query_chunk(run2.cfg, n_q, device="cuda")
    lens = run2.cfg.decode_lens()
    out = _multi(run2, Q, lens)
    stats = _compare(_oracle_multi(oracle, run2, Q, lens), out)
    log_record({"case": f"multi_ctx3000_nq{n_q}", **stats})


def test_multi_token_n1_is_the_decode_bitwise(run2):
    Q = wl.query_chunk(run2.cfg, 1, device="cuda")
    lens = run2.cfg.decode_lens()
    out = _multi(run2, Q, lens)
    _, ref = run2.decode(Q=Q[:, 0].contiguous(), lens=lens)
    torch.cuda.synchronize()
    assert torch.equal(out[:, 0], ref)


def test_multi_token_causal_rows_see_only_their_prefix(run2):
    """Row i must not change when tokens after its position change: compare the chunk's
    rows with single decodes over the matching prefix lengths (same GPU kernels)."""
    n_q = 5
    Q = wl.query_chunk(run2.cfg, n_q, device="cuda")
    L = run2.cfg.decode_lens()[0]
    out = _multi(run2, Q, [L])
    for i in range(n_q):
        _, ref = run2.decode(Q=Q[:, i].contiguous(), lens=[L - n_q + i + 1], max_len=L)
        torch.cuda.synchronize()
        rel = ((out[:, i] - ref).norm() / ref.norm()).item()
        assert rel < 1e-3, (i, rel)   # another kernel: rounding only; a causality error is O(1)


@pytest.mark.parametrize("variant", ["batched_ragged_G4", "gqa1_d128", "gqa16_d128", "d256"])
def test_multi_token_edge_shapes(oracle, variant):
    if variant == "batched_ragged_G4":
        cfg = wl.small_variant(wl.workload(4), n_seqs=4, len_range=(1, 700))
        n_q = 6
    elif variant == "gqa1_d128":
        from dataclasses import replace
        cfg = replace(wl.small_variant(wl.workload(2), length=520), n_q_heads=4)
        n_q = 9
    elif variant == "gqa16_d128":
        from dataclasses import replace
        cfg = replace(wl.small_variant(wl.workload(2), length=333), n_kv_heads=2, n_q_heads=32)
        n_q = 3
    else:
        cfg = wl.small_variant(wl.workload(3), length=400)
        n_q = 5
    run = Run(cfg)
    run.prefill()
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    lens = list(cfg.decode_lens())
    if variant == "batched_ragged_G4":
        lens[0] = 3            # shorter than the chunk: rows 0..2 attend nothing
    out = _multi(run, Q, lens)
    stats = _compare(_oracle_multi(oracle, run, Q, lens), out)
    if variant == "batched_ragged_G4":
        assert torch.all(out[0, :3] == 0)
    log_record({"case": f"multi_{variant}_nq{n_q}", **stats})


def test_multi_token_rejects_bad_arguments(run2):
    lib = iq.raw_lib()
    cfg = run2.cfg
    Q = wl.query_chunk(cfg, 2, device="cuda")
    out = torch.empty((1, 2, cfg.n_q_heads, cfg.d), device="cuda")
    sl = torch.tensor([100], dtype=torch.int32, device="cuda")
    ws = torch.empty((1 << 20,), dtype=torch.uint8, device="cuda")
    args = lambda n_q, nb: (run2.params.handle, iq.ctypes.byref(run2.cache.c), Q.data_ptr(),
                            iq.ISOQ_BF16, 1, n_q, cfg.n_q_heads, sl.data_ptr(), 100,
                            out.data_ptr(), cfg.scale, ws.data_ptr(), nb, None)
    assert lib.isoq_multi_token_attention(*args(0, 1 << 20)) == iq.ISOQ_E_ARG
    need = iq.isoq_multi_token_workspace_bytes(1, 2, cfg.n_q_heads, cfg.n_kv_heads, cfg.d, 100)
    assert lib.isoq_multi_token_attention(*args(2, need - 16)) == iq.ISOQ_E_WORKSPACE
    assert lib.isoq_multi_token_attention(*args(2, need)) == iq.ISOQ_OK
    torch.cuda.synchronize()


# The tensor-memory kernel takes KV heads with >= 128 (query token, head) rows.  These cases
# reach it with ragged batches (a sequence shorter than the chunk), a partial second row
# group, fp32 queries, the 2- and 4-bit formats and a context of several chunks.
@pytest.mark.parametrize("case", ["ragged_G4_nq32", "rows160", "fp32_G4_nq64", "long_20k"])
def test_multi_token_tensor_memory_kernel(oracle, case):
    from dataclasses import replace
    if case == "ragged_G4_nq32":
        cfg = wl.small_variant(wl.workload(4), n_seqs=3, len_range=(40, 1500))
        n_q = 32
    elif case == "rows160":
        cfg = wl.small_variant(wl.workload(2), length=900)
        n_q = 20
    elif case == "fp32_G4_nq64":
        cfg = wl.workload(1)
        n_q = 64
    else:
        cfg = wl.small_variant(wl.workload(2), length=20000)
        n_q = 16
    assert n_q * cfg.n_q_heads // cfg.n_kv_heads >= 128
    run = Run(cfg)
    run.prefill()
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    lens = list(cfg.decode_lens())
    if case == "ragged_G4_nq32":
        lens[0] = 10  # shorter than the chunk: its first 22 query tokens attend nothing
    out = _multi(run, Q, lens)
    stats = _compare(_oracle_multi(oracle, run, Q, lens), out)
    if case == "ragged_G4_nq32":
        assert torch.all(out[0, :22] == 0)
    assert iq.isoq_get_status(run.cache) == 0
    log_record({"case": f"multi_tc_{case}", **stats})


@pytest.mark.parametrize("bits,rot", [(2, 0), (4, 1)])
def test_multi_token_tensor_memory_kernel_formats(oracle, bits, rot):
    cfg = wl.small_variant(wl.workload(2), length=1100)
    run = Run(cfg, bits=bits, rot=rot)
    run.prefill()
    n_q = 16
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    L = cfg.decode_lens()[0]
    out = _multi(run, Q, [L])
    pt = run.layout.page_table.numpy()
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64,
                                  run.cache.blocks.cpu().numpy(), np.repeat(pt[:1], n_q, 0),
                                  [L - n_q + i + 1 for i in range(n_q)],
                                  Q[0].float().cpu().numpy().astype(np.float64), cfg.scale,
                                  bits=bits, rot=rot)
    stats = _compare(ref[None], out)
    log_record({"case": f"multi_tc_b{bits}_r{rot}", **stats})


@pytest.mark.parametrize("n_q", [1, 4, 16])
def test_bad_last_page_is_masked_and_reported(oracle, n_q):
    """A page-table entry outside [0, n_pages) on the last page of a sequence: every kernel
    (per-row decode, shared-page and tensor-memory multi-token) skips the page's tokens and
    sets ISOQ_ST_PAGE_RANGE, so each row equals the oracle over the tokens before that page."""
    cfg = wl.small_variant(wl.workload(2), length=1000)
    run = Run(cfg)
    run.prefill()
    L = cfg.decode_lens()[0]
    last = (L - 1) // 64
    good = last * 64  # tokens before the bad page
    run.cache.page_table[0, last] = -1
    iq.isoq_reset_status(run.cache)
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    out = _multi(run, Q, [L])
    assert iq.isoq_get_status(run.cache) == iq.ISOQ_ST_PAGE_RANGE
    pt = run.layout.page_table.numpy()
    lens_i = [min(L - n_q + i + 1, good) for i in range(n_q)]
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64,
                                  run.cache.blocks.cpu().numpy(), np.repeat(pt[:1], n_q, 0),
                                  lens_i, Q[0].float().cpu().numpy().astype(np.float64),
                                  cfg.scale)
    stats = _compare(ref[None], out)
    log_record({"case": f"multi_bad_last_page_nq{n_q}", **stats})
