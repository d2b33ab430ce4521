"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded
inputs.  Codes bit-exact outside a 1e-6 band around the decision thresholds, binary16
norms within 1 ulp, attention within 2e-3 relative L2 per (sequence, query head) of the
oracle run on the GPU's own packed cache.

Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
Compressed-Space Attention", Abstract.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from _gpu_util import Run, check_attention, check_codes, codes_all, gather_records

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl

pytestmark = pytest.mark.gpu

_LOG = os.environ.get("ISOQ_PARITY_LOG")


def _log(name, stats):
    print(name, json.dumps(stats))
    if _LOG:
        with open(_LOG, "a") as f:
            f.write(json.dumps({"case": name, **stats}) + "\n")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


_codes_all = codes_all


def _all_tokens(cfg):
    seqs, pos = [], []
    for s, n in enumerate(cfg.prefill_lens()):
        seqs.append(np.full(n, s))
        pos.append(np.arange(n))
    return np.concatenate(seqs), np.concatenate(pos)


def _sample_tokens(cfg, per_seq, rng):
    seqs, pos = [], []
    for s, n in enumerate(cfg.prefill_lens()):
        p = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, per_seq)]))
        seqs.append(np.full(len(p), s))
        pos.append(p)
    return np.concatenate(seqs), np.concatenate(pos)


# ------------------------------------------------------------------------------------
# The five workloads
# ------------------------------------------------------------------------------------
def test_config1_full(oracle):
    cfg = wl.workload(1)
    run = Run(cfg)
    run.prefill()
    seqs, pos = _all_tokens(cfg)
    _log("cfg1_codes", _codes_all(oracle, run, seqs, pos))
    Q, out = run.decode()
    _log("cfg1_attention", check_attention(oracle, run, Q, out, cfg.decode_lens()))
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("idx", [2, 3])
def test_config_32k_full(oracle, idx):
    cfg = wl.workload(idx)
    run = Run(cfg)
    run.prefill()
    seqs, pos = _all_tokens(cfg)
    _log(f"cfg{idx}_codes", _codes_all(oracle, run, seqs, pos))
    Q, out = run.decode()
    _log(f"cfg{idx}_attention", check_attention(oracle, run, Q, out, cfg.decode_lens()))
    assert iq.isoq_get_status(run.cache) == 0


def test_config4_batched_paged(oracle):
    cfg = wl.workload(4)
    run = Run(cfg)
    run.prefill()
    K, V, sid, pos = run.append()
    rng = np.random.default_rng(4)
    seqs, p = _sample_tokens(cfg, 24, rng)
    _log("cfg4_codes_sampled", _codes_all(oracle, run, seqs, p))
    # appended tokens: all of them
    kc, kn, vc, vn = gather_records(run.cache, run.layout.page_table, sid.cpu().numpy(),
                                    pos.cpu().numpy(), cfg.d)
    p64 = run.params64()
    sk = check_codes(oracle, p64, K.float().cpu().numpy().astype(np.float64), kc, kn, cfg.d)
    sv = check_codes(oracle, p64, V.float().cpu().numpy().astype(np.float64), vc, vn, cfg.d)
    _log("cfg4_codes_appended", {k: sk[k] + sv[k] for k in sk})
    Q, out = run.decode()
    # every KV head (and so every head's rotation parameters) for the shortest, the longest
    # and a dozen random sequences; the query head inside the group varies
    lens = cfg.decode_lens()
    seqs4 = [int(np.argmin(lens)), int(np.argmax(lens))]
    seqs4 += [int(x) for x in rng.choice([i for i in range(cfg.n_seqs) if i not in seqs4], 12,
                                         replace=False)]
    sel = [(s, kv * cfg.group + (s + kv) % cfg.group) for s in seqs4
           for kv in range(cfg.n_kv_heads)]
    stats = check_attention(oracle, run, Q, out, lens, sel)
    assert stats["pairs"] == 14 * cfg.n_kv_heads
    _log("cfg4_attention_every_kv_head", stats)
    assert iq.isoq_get_status(run.cache) == 0


def test_config5_long_context(oracle):
    cfg = wl.workload(5)
    run = Run(cfg)
    run.prefill()
    rng = np.random.default_rng(5)
    seqs, p = _sample_tokens(cfg, 64, rng)
    _log("cfg5_codes_sampled", _codes_all(oracle, run, seqs, p))
    Q, out = run.decode()
    # one query head of every KV head, for every sequence (the head inside the group varies)
    sel = [(s, kv * cfg.group + (s + kv) % cfg.group) for s in range(cfg.n_seqs)
           for kv in range(cfg.n_kv_heads)]
    stats = check_attention(oracle, run, Q, out, cfg.decode_lens(), sel)
    assert stats["pairs"] == cfg.n_seqs * cfg.n_kv_heads
    _log("cfg5_attention_every_kv_head", stats)
    assert torch.isfinite(out).all()
    assert iq.isoq_get_status(run.cache) == 0


# ------------------------------------------------------------------------------------
# Edge cases
# ------------------------------------------------------------------------------------
def _custom(d=128, n_kv=2, G=4, lens=(1, 63, 64, 65), dtype=torch.float32):
    from dataclasses import replace
    base = wl.workload(1) if d == 128 else wl.workload(3)
    return replace(base, n_seqs=len(lens), n_q_heads=n_kv * G, n_kv_heads=n_kv, d=d,
                   fixed_len=0, len_range=(0, 0), in_dtype=dtype), list(lens)


class _LenRun(Run):
    def prefill(self):
        for s, n in enumerate(self._lens):
            if n == 0:
                continue
            K, V = wl.kv_tokens(self.cfg, s, 0, n, device="cuda")
            sid = torch.full((n,), s, dtype=torch.int32, device="cuda")
            pos = torch.arange(n, dtype=torch.int32, device="cuda")
            iq.isoq_quantize_append(self.params, self.cache, K, V, sid, pos)


def _len_run(cfg, lens):
    """A Run over explicit per-sequence lengths with a shuffled page table."""
    run = _LenRun.__new__(_LenRun)
    run._lens = lens
    run.cfg = cfg
    run.device = "cuda"
    run.bits, run.rot = 3, 0
    run.params = iq.isoq_make_params(wl.PARAM_SEED, cfg.d, cfg.n_kv_heads)
    npg = [max(1, -(-n // 64)) for n in lens]
    rng = np.random.default_rng(sum(lens))
    ids = rng.permutation(sum(npg)).astype(np.int32)
    pt = np.full((len(lens), max(npg)), -1, np.int32)
    o = 0
    for s, n in enumerate(npg):
        pt[s, :n] = ids[o:o + n]
        o += n
    run.layout = wl.PageLayout(torch.from_numpy(pt), int(sum(npg)), [n * 64 for n in npg])
    run.cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, run.layout.n_pages, run.layout.page_table)
    return run


@pytest.mark.parametrize("d,G,lens,hint", [
    (128, 4, (1, 63, 64, 65), None),
    (128, 8, (0, 5, 200, 1000), 4096),        # empty sequence + many empty splits
    (128, 4, (0, 17, 900), None),             # empty sequence, one chunk: no combine
    (128, 1, (129, 3000), None),
    (128, 16, (777,), None),
    (256, 2, (1, 64, 130), None),
    (256, 8, (300, 2049), 8192),
])
def test_edge_lengths(oracle, d, G, lens, hint):
    cfg, lens = _custom(d=d, G=G, lens=lens)
    run = _len_run(cfg, lens)
    run.prefill()
    Q = wl.queries(cfg, device="cuda")
    Q, out = run.decode(Q=Q, lens=lens, max_len=hint or max(lens))
    st = check_attention(oracle, run, Q, out, lens)
    _log(f"edge_d{d}_G{G}_{'-'.join(map(str, lens))}", st)
    for s, n in enumerate(lens):
        if n == 0:
            assert torch.count_nonzero(out[s]) == 0
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("d,G,lens", [(128, 8, (0, 300, 900)), (128, 4, (1, 64, 1000)),
                                      (256, 2, (5, 700))])
def test_single_chunk_output_matches_combine(oracle, d, G, lens):
    """A decode whose contexts fit one chunk writes its output rows from the split kernel
    (normalisation and inverse rotation there, no combine launch).  The same decode planned
    for a longer context (a larger length hint: several chunks, all but the first empty) goes
    through the partials and the combine; the two outputs are bitwise equal."""
    cfg, lens = _custom(d=d, G=G, lens=lens)
    run = _len_run(cfg, lens)
    run.prefill()
    Q = wl.queries(cfg, device="cuda")
    hq = cfg.n_kv_heads * G
    assert iq.isoq_decode_num_splits(len(lens), hq, cfg.n_kv_heads, d, max(lens)) == 1
    assert iq.isoq_decode_num_splits(len(lens), hq, cfg.n_kv_heads, d, 16384) > 1
    Q, direct = run.decode(Q=Q, lens=lens)
    Q, merged = run.decode(Q=Q, lens=lens, max_len=16384)
    assert torch.equal(direct, merged)
    _log(f"direct_d{d}_G{G}_{'-'.join(map(str, lens))}",
         check_attention(oracle, run, Q, direct, lens))
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("kv_dtype,q_dtype", [(torch.float16, torch.float16),
                                              (torch.bfloat16, torch.float32),
                                              (torch.float32, torch.bfloat16)])
def test_dtypes(oracle, kv_dtype, q_dtype):
    cfg, lens = _custom(lens=(100, 257), dtype=kv_dtype)
    run = _len_run(cfg, lens)
    run.prefill()
    seqs = np.concatenate([np.full(n, s) for s, n in enumerate(lens)])
    pos = np.concatenate([np.arange(n) for n in lens])
    _log(f"dtype_{kv_dtype}_codes", _codes_all(oracle, run, seqs, pos))
    Q = wl.queries(cfg, device="cuda").to(q_dtype)
    Q, out = run.decode(Q=Q, lens=lens)
    _log(f"dtype_{kv_dtype}_{q_dtype}_attention", check_attention(oracle, run, Q, out, lens))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n_kv,lens", [(3, (1, 127, 128, 129)), (1, (255, 300)), (8, (513,)),
                                       (8, (1300, 1281)), (5, (2000,))])
def test_quantize_tiles(oracle, dtype, n_kv, lens):
    """16-bit appends at d = 128 transform 128-token tiles on the tensor cores: lengths around
    the tile size, an odd head count, several tiles per sequence and per CTA."""
    cfg, lens = _custom(n_kv=n_kv, G=2, lens=lens, dtype=dtype)
    run = _len_run(cfg, lens)
    run.prefill()
    seqs = np.concatenate([np.full(n, s) for s, n in enumerate(lens)])
    pos = np.concatenate([np.arange(n) for n in lens])
    _log(f"tiles_{dtype}_H{n_kv}_{'-'.join(map(str, lens))}", _codes_all(oracle, run, seqs, pos))
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n_kv,lens", [(2, (150, 200)), (8, (1500, 1200))])
def test_quantize_tiles_mixed_tokens(oracle, dtype, n_kv, lens):
    """One append whose tiles mix sequences and positions in shuffled order."""
    cfg, lens = _custom(n_kv=n_kv, G=2, lens=lens, dtype=dtype)
    run = _len_run(cfg, lens)
    Ks, Vs, sids, poss = [], [], [], []
    for s, n in enumerate(lens):
        K, V = wl.kv_tokens(cfg, s, 0, n, device="cuda")
        Ks.append(K)
        Vs.append(V)
        sids.append(torch.full((n,), s, dtype=torch.int32))
        poss.append(torch.arange(n, dtype=torch.int32))
    perm = torch.from_numpy(np.random.default_rng(7).permutation(sum(lens)))
    K = torch.cat(Ks)[perm.cuda()].contiguous()
    V = torch.cat(Vs)[perm.cuda()].contiguous()
    sid = torch.cat(sids)[perm].cuda()
    pos = torch.cat(poss)[perm].cuda()
    iq.isoq_quantize_append(run.params, run.cache, K, V, sid, pos)
    seqs = np.concatenate([np.full(n, s) for s, n in enumerate(lens)])
    p = np.concatenate([np.arange(n) for n in lens])
    _log(f"tiles_mixed_{dtype}_H{n_kv}", _codes_all(oracle, run, seqs, p))
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_vector_and_norm_saturation(oracle, dtype):
    cfg, lens = _custom(lens=(70,), dtype=dtype)
    run = _len_run(cfg, lens)
    K, V = wl.kv_tokens(cfg, 0, 0, 70, device="cuda")
    K[3] = 0.0          # zero vectors -> codes 4, norm 0
    V[5] = 0.0
    K[7] *= 1e5         # norm > 65504 -> saturates to 65504, status bit
    sid = torch.zeros(70, dtype=torch.int32, device="cuda")
    pos = torch.arange(70, dtype=torch.int32, device="cuda")
    iq.isoq_quantize_append(run.params, run.cache, K, V, sid, pos)
    kc, kn, vc, vn = gather_records(run.cache, run.layout.page_table, np.zeros(70, int),
                                    np.arange(70), cfg.d)
    codes = oracle.unpack_codes_batch(kc, cfg.d)
    assert np.all(codes[3] == 4) and np.all(kn[3] == 0)
    assert np.all(oracle.unpack_codes_batch(vc, cfg.d)[5] == 4) and np.all(vn[5] == 0)
    assert np.all(kn[7] == 0x7BFF)
    assert iq.isoq_get_status(run.cache) == iq.ISOQ_ST_NORM_SAT
    p64 = run.params64()
    st = check_codes(oracle, p64, K.float().cpu().numpy().astype(np.float64), kc, kn, cfg.d)
    _log("zero_and_saturation", st)
    iq.isoq_reset_status(run.cache)
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_out_of_range_writes_are_skipped(dtype):
    cfg, lens = _custom(lens=(64, 64), dtype=dtype)
    run = _len_run(cfg, lens)
    K, V = wl.kv_tokens(cfg, 0, 0, 4, device="cuda")
    before = run.cache.blocks.clone()
    cases = [([2], [0], iq.ISOQ_ST_SEQ_RANGE), ([-1], [0], iq.ISOQ_ST_SEQ_RANGE),
             ([0], [64], iq.ISOQ_ST_POS_RANGE), ([1], [-1], iq.ISOQ_ST_POS_RANGE)]
    for s, p, bit in cases:
        iq.isoq_reset_status(run.cache)
        sid = torch.tensor(s, dtype=torch.int32, device="cuda")
        pos = torch.tensor(p, dtype=torch.int32, device="cuda")
        iq.isoq_quantize_append(run.params, run.cache, K[:1], V[:1], sid, pos)
        assert iq.isoq_get_status(run.cache) == bit
        assert torch.equal(run.cache.blocks, before)
    # a page-table entry outside [0, n_pages)
    run.cache.page_table[1, 0] = run.layout.n_pages
    iq.isoq_reset_status(run.cache)
    iq.isoq_quantize_append(run.params, run.cache, K[:1], V[:1],
                            torch.tensor([1], dtype=torch.int32, device="cuda"),
                            torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert iq.isoq_get_status(run.cache) == iq.ISOQ_ST_PAGE_RANGE
    assert torch.equal(run.cache.blocks, before)


def test_decode_len_beyond_capacity_is_clamped(oracle):
    cfg, lens = _custom(lens=(100,))
    run = _len_run(cfg, lens)
    run.prefill()
    Q = wl.queries(cfg, device="cuda")
    # capacity is 2 pages = 128 tokens; ask for 200 -> clamped to 128 (slots 100..127 are
    # zero-initialised codes with norm 0)
    Q, out = run.decode(Q=Q, lens=[200], max_len=200)
    assert iq.isoq_get_status(run.cache) == iq.ISOQ_ST_LEN_RANGE
    check_attention(oracle, run, Q, out, [128])


def test_deterministic():
    cfg, lens = _custom(lens=(500, 33))
    run = _len_run(cfg, lens)
    run.prefill()
    b1 = run.cache.blocks.clone()
    run.prefill()
    assert torch.equal(run.cache.blocks, b1)
    Q = wl.queries(cfg, device="cuda")
    _, o1 = run.decode(Q=Q, lens=lens)
    _, o2 = run.decode(Q=Q, lens=lens)
    assert torch.equal(o1, o2)


def test_error_codes():
    cfg, lens = _custom(lens=(64,))
    run = _len_run(cfg, lens)
    Q = wl.queries(cfg, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.empty((1, cfg.n_q_heads, cfg.d), device="cuda")
    nb = iq.isoq_decode_workspace_bytes(1, cfg.n_q_heads, cfg.n_kv_heads, cfg.d, 64)
    ws = torch.empty((nb,), dtype=torch.uint8, device="cuda")
    with pytest.raises(iq.IsoqError) as e:
        iq.isoq_decode_attention(run.params, run.cache, Q, sl, 64, out, cfg.scale, ws[:nb - 16])
    assert e.value.code == iq.ISOQ_E_WORKSPACE
    with pytest.raises(iq.IsoqError) as e:      # 6 query heads over 2 KV heads is fine; 7 is not
        iq.isoq_decode_attention(run.params, run.cache, Q[:, :7].contiguous(), sl, 64,
                                 out[:, :7].contiguous(), cfg.scale, ws)
    assert e.value.code == iq.ISOQ_E_GQA
    with pytest.raises(iq.IsoqError) as e:      # params of another head count
        p2 = iq.isoq_make_params(0, cfg.d, cfg.n_kv_heads + 1)
        K, V = wl.kv_tokens(cfg, 0, 0, 1, device="cuda")
        iq.isoq_quantize_append(p2, run.cache, K, V, sl[:1] * 0, sl[:1] * 0)
    assert e.value.code == iq.ISOQ_E_DIM
    with pytest.raises(iq.IsoqError) as e:
        iq.isoq_make_params(0, 96, 2)
    assert e.value.code == iq.ISOQ_E_DIM
    # K, V must start on a 16-byte boundary (rejected before any launch; cache untouched)
    K, V = wl.kv_tokens(cfg, 0, 0, 3, device="cuda")
    flat = torch.empty(K.numel() + 8, dtype=K.dtype, device="cuda")
    Kmis = flat[1:1 + K.numel()].view(K.shape)
    Kmis.copy_(K)
    before = run.cache.blocks.clone()
    with pytest.raises(iq.IsoqError) as e:
        iq.isoq_quantize_append(run.params, run.cache, Kmis, V, sl[:1].repeat(3) * 0,
                                torch.arange(3, dtype=torch.int32, device="cuda"))
    assert e.value.code == iq.ISOQ_E_ARG
    assert torch.equal(run.cache.blocks, before)
    lib = iq.raw_lib()
    import ctypes
    assert lib.isoq_decode_attention(run.params.handle, ctypes.byref(run.cache.c), None, 0, 1,
                                     cfg.n_q_heads, sl.data_ptr(), 64, out.data_ptr(),
                                     cfg.scale, ws.data_ptr(), nb, None) == iq.ISOQ_E_ARG
    assert lib.isoq_decode_attention(run.params.handle, ctypes.byref(run.cache.c),
                                     Q.data_ptr(), 7, 1, cfg.n_q_heads, sl.data_ptr(), 64,
                                     out.data_ptr(), cfg.scale, ws.data_ptr(), nb,
                                     None) == iq.ISOQ_E_ARG
    assert lib.isoq_decode_attention(run.params.handle, ctypes.byref(run.cache.c),
                                     Q.data_ptr(), 0, 1, cfg.n_q_heads, sl.data_ptr(), 64,
                                     out.data_ptr(), float("nan"), ws.data_ptr(), nb,
                                     None) == iq.ISOQ_E_ARG
    # nothing above launched a kernel that failed
    torch.cuda.synchronize()
    assert iq.isoq_last_cuda_error() == 0
