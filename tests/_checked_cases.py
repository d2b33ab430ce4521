"""Runs the CUDA path of the bounds-checked build (libisoq_checked.so) on a handful of
workloads and checks each against the oracle.  Executed as a child process by
test_gpu_bounds_checked.py, with ISOQ_CHECK_BOUNDS=1 so that the package loads the checked
library:

    ISOQ_CHECK_BOUNDS=1 python tests/_checked_cases.py [case ...]

Cases: the 1024-token GQA-4 workload (every code, every head), the 32k-token d = 256
workload (sampled codes, every head), a ragged batch of the 64-sequence paged workload
with single-token appends (every KV head of every sequence), the two multi-token kernels,
the 2- and 4-bit formats (both rotation forms), and the RoPE-fused and layer-batched
quantize-appends.  Each case must leave the cache's status word at 0 (no index outside its extent,
no other condition) and stay within the parity tolerances.  One JSON line per case; exit
status 0 when all pass.
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import rotated_bit_kv_isoquant_b200 as iq  # noqa: E402
import workloads as wl  # noqa: E402
from _gpu_util import Run, check_attention, codes_all  # noqa: E402


def _tokens(cfg, per_seq=None, seed=0):
    rng = np.random.default_rng(seed)
    seqs, pos = [], []
    for s, n in enumerate(cfg.prefill_lens()):
        p = np.arange(n) if per_seq is None else np.unique(
            np.concatenate([[0, n - 1], rng.integers(0, n, per_seq)]))
        seqs.append(np.full(len(p), s))
        pos.append(p)
    return np.concatenate(seqs), np.concatenate(pos)


def _status(run):
    return iq.isoq_get_status(run.cache)


def case_cfg1(oracle):
    cfg = wl.workload(1)
    run = Run(cfg)
    run.prefill()
    seqs, pos = _tokens(cfg)
    codes = codes_all(oracle, run, seqs, pos)
    Q, out = run.decode()
    att = check_attention(oracle, run, Q, out, cfg.decode_lens())
    return {"codes": codes, "attention": att, "status": _status(run)}


def case_cfg3(oracle):
    cfg = wl.workload(3)
    run = Run(cfg)
    run.prefill()
    seqs, pos = _tokens(cfg, per_seq=512, seed=3)
    codes = codes_all(oracle, run, seqs, pos)
    Q, out = run.decode()
    att = check_attention(oracle, run, Q, out, cfg.decode_lens())
    return {"codes": codes, "attention": att, "status": _status(run)}


def case_ragged(oracle):
    cfg = wl.small_variant(wl.workload(4), n_seqs=12, len_range=(1, 3000))
    run = Run(cfg)
    run.prefill()
    run.append()
    seqs, pos = _tokens(cfg, per_seq=48, seed=4)
    codes = codes_all(oracle, run, seqs, pos)
    Q, out = run.decode()
    lens = cfg.decode_lens()
    sel = [(s, kv * cfg.group + (s + kv) % cfg.group) for s in range(cfg.n_seqs)
           for kv in range(cfg.n_kv_heads)]
    att = check_attention(oracle, run, Q, out, lens, sel)
    return {"codes": codes, "attention": att, "status": _status(run),
            "lens": [int(min(lens)), int(max(lens))]}


def _multi_case(oracle, cfg, n_q, lens_edit=None):
    run = Run(cfg)
    run.prefill()
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    lens = list(cfg.decode_lens())
    if lens_edit:
        lens = lens_edit(lens)
    n_seqs, hq = Q.shape[0], Q.shape[2]
    max_len = max(lens)
    nb = iq.isoq_multi_token_workspace_bytes(n_seqs, n_q, hq, cfg.n_kv_heads, cfg.d, max_len)
    ws = torch.empty((max(nb, 16),), dtype=torch.uint8, device="cuda")
    out = torch.empty((n_seqs, n_q, hq, cfg.d), dtype=torch.float32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    iq.isoq_multi_token_attention(run.params, run.cache, Q, sl, max_len, out, cfg.scale, ws)
    torch.cuda.synchronize()
    pt = run.layout.page_table.numpy()
    rows = [(s, i) for s in range(n_seqs) for i in range(n_q)]
    vlen = [max(0, lens[s] - n_q + i + 1) for s, i in rows]
    q = Q.float().cpu().numpy().astype(np.float64).reshape(n_seqs * n_q, hq, cfg.d)
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64,
                                  run.cache.blocks.cpu().numpy(),
                                  np.stack([pt[s] for s, _ in rows]), vlen, q, cfg.scale)
    r = ref.reshape(-1, cfg.d)
    g = out.cpu().numpy().astype(np.float64).reshape(-1, cfg.d)
    nr = np.linalg.norm(r, axis=1)
    nz = nr > 0
    assert np.all(np.isfinite(g)), "non-finite output"
    assert np.all(np.linalg.norm(g[~nz], axis=1) == 0)
    err = np.linalg.norm(g[nz] - r[nz], axis=1) / nr[nz]
    from _gpu_util import ATTN_TOL
    assert err.max() <= ATTN_TOL, f"max rel L2 {err.max()}"
    return {"attention": {"rows": int(r.shape[0]), "max_rel": float(err.max())},
            "status": _status(run)}


def case_multi_mq(oracle):
    # 7 query tokens x GQA 4 = 28 rows per KV head: the register-tile multi-token kernel
    return _multi_case(oracle, wl.small_variant(wl.workload(2), length=2500), 7)


def case_multi_tc(oracle):
    # 32 tokens x GQA 4 = 128 rows, ragged lengths, one shorter than the chunk: the
    # tensor-memory multi-token kernel
    cfg = wl.small_variant(wl.workload(4), n_seqs=3, len_range=(40, 1500))

    def edit(lens):
        lens[0] = 10
        return lens
    return _multi_case(oracle, cfg, 32, edit)


def case_formats(oracle):
    # the 2- and 4-bit formats (the f16 decode kernel) with both rotation forms
    recs = {}
    for bits, rot in ((2, 0), (4, 1)):
        cfg = wl.small_variant(wl.workload(2), length=1100)
        run = Run(cfg, bits=bits, rot=rot)
        run.prefill()
        seqs, pos = _tokens(cfg, per_seq=256, seed=bits)
        codes = codes_all(oracle, run, seqs, pos)
        Q, out = run.decode()
        att = check_attention(oracle, run, Q, out, cfg.decode_lens())
        recs[f"b{bits}_r{rot}"] = {"codes": codes, "attention": att, "status": _status(run)}
    return {"formats": recs, "status": max(r["status"] for r in recs.values())}


def case_rope_layers(oracle):
    # RoPE fused into the per-thread quantizer (a prefill and a decode step's appends), and
    # the layer-batched append of the same step into three caches
    from _gpu_util import check_codes, gather_records
    cfg = wl.small_variant(wl.workload(4), n_seqs=4, len_range=(64, 700))
    lay = wl.page_layout(cfg)
    lens = cfg.prefill_lens()
    tab = iq.isoq_rope_table(cfg.d, max(lens) + 1)
    params = [iq.isoq_make_params(wl.PARAM_SEED + l, cfg.d, cfg.n_kv_heads) for l in range(3)]
    caches = [iq.PagedCache(cfg.d, cfg.n_kv_heads, lay.n_pages, lay.page_table) for _ in range(3)]
    for s, n in enumerate(lens):
        K, V = wl.kv_tokens(cfg, s, 0, n, device="cuda", rope=False)
        sid = torch.full((n,), s, dtype=torch.int32, device="cuda")
        pos = torch.arange(n, dtype=torch.int32, device="cuda")
        iq.isoq_quantize_append_rope(params[0], caches[0], K, V, sid, pos, tab)
    sid = torch.arange(cfg.n_seqs, dtype=torch.int32, device="cuda")
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    Ks = [torch.randn((cfg.n_seqs, cfg.n_kv_heads, cfg.d), generator=g, device="cuda").bfloat16()
          for _ in range(3)]
    Vs = [torch.randn((cfg.n_seqs, cfg.n_kv_heads, cfg.d), generator=g, device="cuda").bfloat16()
          for _ in range(3)]
    iq.isoq_quantize_append_layers(params, caches, Ks, Vs, sid, pos, rope_table=tab)
    torch.cuda.synchronize()
    # the prefill codes of sequence 0 against the oracle's RoPE and quantiser
    n0 = lens[0]
    K0, V0 = wl.kv_tokens(cfg, 0, 0, n0, device="cuda", rope=False)
    kc, kn, vc, vn = gather_records(caches[0], lay.page_table, np.zeros(n0, int), np.arange(n0),
                                    cfg.d)
    _, p32 = oracle.make_params_v(wl.PARAM_SEED, cfg.d, cfg.n_kv_heads, 0)
    p64 = p32.astype(np.float64)
    Kr = oracle.rope(K0.float().cpu().numpy().astype(np.float64),
                     np.repeat(np.arange(n0), cfg.n_kv_heads), 10000.0)
    sk = check_codes(oracle, p64, Kr, kc, kn, cfg.d)
    sv = check_codes(oracle, p64, V0.float().cpu().numpy().astype(np.float64), vc, vn, cfg.d)
    st = max(iq.isoq_get_status(c) for c in caches)
    return {"codes": {k: sk[k] + sv[k] for k in sk}, "status": st}


CASES = {"cfg1": case_cfg1, "cfg3": case_cfg3, "ragged": case_ragged,
         "multi_mq": case_multi_mq, "multi_tc": case_multi_tc, "formats": case_formats,
         "rope_layers": case_rope_layers}


def main(names):
    import oracle
    oracle.build()
    assert iq.CHECKED, "set ISOQ_CHECK_BOUNDS=1: this runner is for the bounds-checked build"
    assert os.path.basename(iq.LIB_PATH) == "libisoq_checked.so"
    torch.cuda.set_device(0)
    st = iq.isoq_selftest_bounds()
    print(json.dumps({"case": "selftest", "status": st}), flush=True)
    failed = st != iq.ISOQ_ST_BOUNDS
    for name in names or list(CASES):
        try:
            rec = CASES[name](oracle)
            ok = rec["status"] == 0
        except AssertionError as e:
            rec, ok = {"error": str(e)}, False
        print(json.dumps({"case": name, "ok": ok, **rec}), flush=True)
        failed |= not ok
    return 1 if failed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
