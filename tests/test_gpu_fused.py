"""Fused epilogues on the GPU: RoPE applied to K inside quantize-append (against the fp64
oracle's RoPE followed by its quantiser), the device RoPE table (against numpy's fp64
cos/sin), and layer-batched appends (bitwise equal to one append per layer)."""
import numpy as np
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl
from _gpu_util import Run, check_attention, check_codes, gather_records, log_record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("d", [128, 256])
def test_rope_table_matches_fp64(d):
    max_pos = 70000
    t = iq.isoq_rope_table(d, max_pos).cpu().numpy().astype(np.float64)
    pos = np.array([0, 1, 2, 17, 4095, 65536, 69999])
    theta = 10000.0 ** (-2.0 * np.arange(d // 2) / d)
    ang = pos[:, None] * theta[None, :]
    assert np.abs(t[pos, :, 0] - np.cos(ang)).max() < 2e-7      # binary32 rounding
    assert np.abs(t[pos, :, 1] - np.sin(ang)).max() < 2e-7


@pytest.mark.parametrize("cfg_idx,bits,rot", [(3, 3, 0), (2, 3, 0), (2, 4, 1)])
def test_fused_rope_quantize_matches_oracle(oracle, cfg_idx, bits, rot):
    base_cfg = wl.workload(cfg_idx)
    cfg = wl.small_variant(base_cfg, length=900)
    run = Run(cfg, bits=bits, rot=rot)
    L = cfg.prefill_lens()[0]
    start = 4992                                 # page-aligned, beyond the first 4096 positions
    from dataclasses import replace
    tab = iq.isoq_rope_table(cfg.d, start + L + 64)
    # the cache holds positions start .. start+L-1 of sequence 0: a page table long enough
    n_pages = -(-(start + L) // 64)
    pt = torch.arange(n_pages, dtype=torch.int32)[None, :]
    run.cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, n_pages, pt, bits=bits)
    run.layout = replace(run.layout, page_table=pt, n_pages=n_pages)
    K, V = wl.kv_tokens(cfg, 0, 0, L, device="cuda", rope=False)
    sid = torch.zeros((L,), dtype=torch.int32, device="cuda")
    pos = torch.arange(start, start + L, dtype=torch.int32, device="cuda")
    iq.isoq_quantize_append_rope(run.params, run.cache, K, V, sid, pos, tab)
    torch.cuda.synchronize()
    assert iq.isoq_get_status(run.cache) == 0
    positions = np.arange(start, start + L)
    kc, kn, vc, vn = gather_records(run.cache, pt, np.zeros(L, int), positions, cfg.d, bits)
    Kr = oracle.rope(K.float().cpu().numpy().astype(np.float64),
                     np.repeat(positions, cfg.n_kv_heads), 10000.0)
    p64 = run.params64()
    sk = check_codes(oracle, p64, Kr, kc, kn, cfg.d, bits, rot)
    sv = check_codes(oracle, p64, V.float().cpu().numpy().astype(np.float64), vc, vn, cfg.d,
                     bits, rot)
    log_record({"case": f"fused_rope_cfg{cfg_idx}_b{bits}_r{rot}",
                **{k: sk[k] + sv[k] for k in sk}})
    # decode over the filled pages only (a view whose page table starts at position start)
    view_pt = pt[:, start // 64:].clone()
    run.layout = replace(run.layout, page_table=view_pt)
    run.cache = _View(run.cache, view_pt)
    Q, out = run.decode(lens=[L])
    torch.cuda.synchronize()
    log_record({"case": f"fused_rope_decode_cfg{cfg_idx}_b{bits}_r{rot}",
                **check_attention(oracle, run, Q, out, [L])})


class _View:
    def __init__(self, base, page_table):
        from rotated_bit_kv_isoquant_b200.context_parallel import CacheSlice
        self._s = CacheSlice(base, page_table)
        self.blocks, self.d, self.n_kv_heads, self.bits = base.blocks, base.d, base.n_kv_heads, base.bits

    @property
    def c(self):
        return self._s.c


def test_fused_rope_rejects_positions_beyond_the_table():
    cfg = wl.small_variant(wl.workload(2), length=128)
    run = Run(cfg)
    tab = iq.isoq_rope_table(cfg.d, 100)
    K, V = wl.kv_tokens(cfg, 0, 0, 128, device="cuda")
    sid = torch.zeros((128,), dtype=torch.int32, device="cuda")
    pos = torch.arange(128, dtype=torch.int32, device="cuda")
    before = run.cache.blocks.clone()
    iq.isoq_quantize_append_rope(run.params, run.cache, K, V, sid, pos, tab)
    torch.cuda.synchronize()
    assert iq.isoq_get_status(run.cache) & iq.ISOQ_ST_POS_RANGE
    # tokens 100..127 were skipped: their slots (page 1, slots 36..63) are untouched
    page1 = run.layout.page_table[0, 1].item()
    assert torch.equal(run.cache.blocks[page1, :, 36 * 48:64 * 48], before[page1, :, 36 * 48:64 * 48])


@pytest.mark.parametrize("n_layers,bits", [(3, 3), (33, 2)])
def test_layer_batched_append_equals_per_layer_appends(n_layers, bits):
    cfg = wl.small_variant(wl.workload(4), n_seqs=4, len_range=(64, 300))
    lay = wl.page_layout(cfg)
    params = [iq.isoq_make_params(100 + l, cfg.d, cfg.n_kv_heads, bits=bits) for l in range(n_layers)]
    batched = [iq.PagedCache(cfg.d, cfg.n_kv_heads, lay.n_pages, lay.page_table, bits=bits)
               for _ in range(n_layers)]
    single = [iq.PagedCache(cfg.d, cfg.n_kv_heads, lay.n_pages, lay.page_table, bits=bits)
              for _ in range(n_layers)]
    # one decode step: one new token per sequence, at position len
    lens = cfg.prefill_lens()
    sid = torch.arange(cfg.n_seqs, dtype=torch.int32, device="cuda")
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    Ks = [torch.randn((cfg.n_seqs, cfg.n_kv_heads, cfg.d), generator=g, device="cuda").bfloat16()
          for _ in range(n_layers)]
    Vs = [torch.randn((cfg.n_seqs, cfg.n_kv_heads, cfg.d), generator=g, device="cuda").bfloat16()
          for _ in range(n_layers)]
    tab = iq.isoq_rope_table(cfg.d, max(lens) + 1)
    iq.isoq_quantize_append_layers(params, batched, Ks, Vs, sid, pos, rope_table=tab)
    for l in range(n_layers):
        iq.isoq_quantize_append_rope(params[l], single[l], Ks[l], Vs[l], sid, pos, tab)
    torch.cuda.synchronize()
    for l in range(n_layers):
        assert torch.equal(batched[l].blocks, single[l].blocks), l
        assert iq.isoq_get_status(batched[l]) == 0


def test_layer_batched_rejects_mixed_formats():
    cfg = wl.small_variant(wl.workload(2), length=64)
    lay = wl.page_layout(cfg)
    p3 = iq.isoq_make_params(0, cfg.d, cfg.n_kv_heads, bits=3)
    p4 = iq.isoq_make_params(0, cfg.d, cfg.n_kv_heads, bits=4)
    c3 = iq.PagedCache(cfg.d, cfg.n_kv_heads, lay.n_pages, lay.page_table, bits=3)
    c4 = iq.PagedCache(cfg.d, cfg.n_kv_heads, lay.n_pages, lay.page_table, bits=4)
    K, V = wl.kv_tokens(cfg, 0, 0, 64, device="cuda")
    sid = torch.zeros((64,), dtype=torch.int32, device="cuda")
    pos = torch.arange(64, dtype=torch.int32, device="cuda")
    with pytest.raises(iq.IsoqError) as e:
        iq.isoq_quantize_append_layers([p3, p4], [c3, c4], [K, K], [V, V], sid, pos)
    assert e.value.code == iq.ISOQ_E_DIM
    with pytest.raises(iq.IsoqError) as e:       # a 4-bit cache with 3-bit params
        iq.isoq_quantize_append(p3, c4, K, V, sid, pos)
    assert e.value.code == iq.ISOQ_E_DIM
