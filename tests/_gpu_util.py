"""Shared helpers of the GPU tests: run the CUDA path on a workload and compare it with the
fp64 oracle (which only ever sees host copies of the same seeded inputs)."""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl

BAND = 1e-6          # codes may differ only where u is this close to a threshold (N(0,1) units)
ATTN_TOL = 2e-3      # relative L2 error per (sequence, query head) vs the oracle on the same codes


def log_record(record: dict) -> None:
    """Print a parity record and append it to $ISOQ_PARITY_LOG (JSON lines) when set."""
    print(json.dumps(record))
    path = os.environ.get("ISOQ_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(record) + "\n")


class Run:
    """One workload on the GPU: params, cache, prefill, appended tokens, decode."""

    def __init__(self, cfg: wl.Workload, device="cuda", seed: int = wl.PARAM_SEED,
                 bits: int = 3, rot: int = 0):
        self.cfg = cfg
        self.device = device
        self.bits, self.rot = bits, rot
        self.params = iq.isoq_make_params(seed, cfg.d, cfg.n_kv_heads, bits=bits, rotation=rot)
        self.layout = wl.page_layout(cfg)
        self.cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, self.layout.n_pages,
                                   self.layout.page_table, device=device, bits=bits)

    def prefill(self):
        cfg = self.cfg
        for s, start, count in wl.prefill_calls(cfg):
            K, V = wl.kv_tokens(cfg, s, start, count, device=self.device)
            sid = torch.full((count,), s, dtype=torch.int32, device=self.device)
            pos = torch.arange(start, start + count, dtype=torch.int32, device=self.device)
            iq.isoq_quantize_append(self.params, self.cache, K, V, sid, pos)

    def append(self):
        K, V, sid, pos = wl.append_kv(self.cfg, device=self.device)
        if K.shape[0]:
            iq.isoq_quantize_append(self.params, self.cache, K, V, sid, pos)
        return K, V, sid, pos

    def decode(self, Q=None, lens=None, max_len=None):
        cfg = self.cfg
        Q = wl.queries(cfg, device=self.device) if Q is None else Q
        lens = cfg.decode_lens() if lens is None else lens
        max_len = max(lens) if max_len is None else max_len
        sl = torch.tensor(lens, dtype=torch.int32, device=self.device)
        out = torch.empty((Q.shape[0], Q.shape[1], cfg.d), dtype=torch.float32, device=self.device)
        nb = iq.isoq_decode_workspace_bytes(Q.shape[0], Q.shape[1], cfg.n_kv_heads, cfg.d, max_len)
        ws = torch.empty((max(nb, 16),), dtype=torch.uint8, device=self.device)
        iq.isoq_decode_attention(self.params, self.cache, Q, sl, max_len, out, cfg.scale, ws)
        return Q, out

    def params64(self):
        """The oracle's own parameters (binary32 values promoted), for the parity path."""
        import oracle
        _, p32 = oracle.make_params_v(wl.PARAM_SEED, self.cfg.d, self.cfg.n_kv_heads, self.rot)
        return p32.astype(np.float64)


def gather_records(cache: iq.PagedCache, page_table: torch.Tensor, seqs, positions, d: int,
                   bits: int = 3):
    """Device -> host: per (token, KV head) the packed K codes, K norm, V codes, V norm.
    Returns (kcodes [n][H][bits*d/8], knorm [n][H], vcodes, vnorm) as numpy."""
    dev = cache.blocks.device
    cb = bits * d // 8
    seqs = torch.as_tensor(np.asarray(seqs), dtype=torch.long, device=dev)
    positions = torch.as_tensor(np.asarray(positions), dtype=torch.long, device=dev)
    pt = page_table.to(dev).long()
    phys = pt[seqs, positions // 64]
    slot = positions % 64
    ar = torch.arange(cb, device=dev)
    k_norm_off, v_codes_off = 64 * cb, 64 * (cb + 2)
    v_norm_off = v_codes_off + 64 * cb
    H = cache.n_kv_heads
    hh = torch.arange(H, device=dev)

    def take(col):  # col: [n][w] byte offsets -> [n][H][w]
        return cache.blocks[phys[:, None, None], hh[None, :, None], col[:, None, :]]

    kc = take(slot[:, None] * cb + ar)
    if bits == 3:
        # 3-bit V codes use the V tile layout: fetch the V regions of the pages involved
        # and let the oracle turn them into per-slot records
        import oracle
        uniq, inv = torch.unique(phys, return_inverse=True)
        reg = cache.blocks[uniq][:, :, v_codes_off:v_codes_off + 64 * cb]
        rec = oracle.v_region_records(reg.cpu().numpy(), d, bits=bits)   # [U][H][64][cb]
        vc = rec[inv.cpu().numpy()[:, None], np.arange(H)[None, :], slot.cpu().numpy()[:, None]]
    else:
        vc = take(v_codes_off + slot[:, None] * cb + ar).cpu().numpy()
    two = torch.arange(2, device=dev)
    kn = take(k_norm_off + 2 * slot[:, None] + two)
    vn = take(v_norm_off + 2 * slot[:, None] + two)
    to16 = lambda t: t.cpu().numpy().copy().view(np.uint16)[..., 0]
    return kc.cpu().numpy(), to16(kn), vc, to16(vn)


def check_codes(oracle, params64, X, gpu_codes_packed, gpu_norms, d, bits: int = 3, rot: int = 0):
    """Compare GPU packed codes / norms of X ([n][H][d] host) with the oracle.
    Returns a dict of statistics; raises AssertionError on a violation."""
    codes, norms, dist = oracle.quantize_rows(params64, X, bits=bits, rot=rot)
    g = oracle.unpack_codes_batch(gpu_codes_packed, d, bits=bits)
    diff = g != codes
    n_diff = int(diff.sum())
    in_band = dist < BAND
    if n_diff:
        assert np.all(in_band[diff]), (
            f"{int((diff & ~in_band).sum())} code mismatches outside the {BAND} band; "
            f"max dist {dist[diff].max()}")
        assert np.all(np.abs(g[diff].astype(int) - codes[diff].astype(int)) == 1)
    nd = np.abs(gpu_norms.astype(np.int64) - norms.astype(np.int64))
    assert nd.max(initial=0) <= 1, f"norm mismatch > 1 ulp: {nd.max()}"
    return {"vectors": int(X.shape[0] * X.shape[1]), "elements": int(diff.size),
            "mismatch": n_diff, "band": int(in_band.sum()), "norm_ulp_diff": int((nd > 0).sum())}


def check_attention(oracle, run: Run, Q, out, lens, sel=None):
    """Oracle decode on the GPU's own packed cache (host copy) vs the GPU output."""
    cfg = run.cfg
    blocks = run.cache.blocks.cpu().numpy()
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64, blocks,
                                  run.layout.page_table.numpy(), lens,
                                  Q.float().cpu().numpy().astype(np.float64), cfg.scale, sel=sel,
                                  bits=run.bits, rot=run.rot)
    got = out.cpu().numpy().astype(np.float64)
    pairs = sel if sel is not None else [(s, h) for s in range(Q.shape[0])
                                         for h in range(Q.shape[1])]
    errs = []
    for s, h in pairs:
        r, g = ref[s, h], got[s, h]
        nr = np.linalg.norm(r)
        if nr == 0:
            assert np.linalg.norm(g) == 0
            errs.append(0.0)
            continue
        errs.append(float(np.linalg.norm(g - r) / nr))
    errs = np.array(errs)
    assert np.all(np.isfinite(got)), "non-finite output"
    assert errs.max() <= ATTN_TOL, f"max rel L2 {errs.max()} > {ATTN_TOL}"
    return {"pairs": len(pairs), "max_rel": float(errs.max()), "mean_rel": float(errs.mean())}


def codes_all(oracle, run, seqs, positions):
    """Check K and V codes of the given tokens against the oracle."""
    cfg = run.cfg
    kc, kn, vc, vn = gather_records(run.cache, run.layout.page_table, seqs, positions, cfg.d,
                                    run.bits)
    # regenerate the same inputs (chunked seeds) on the device, copy to host
    Ks, Vs = [], []
    order = np.lexsort((positions, seqs))
    assert np.array_equal(order, np.arange(len(order))), "tokens must be sorted by (seq, pos)"
    for s in np.unique(seqs):
        p = np.asarray(positions)[np.asarray(seqs) == s]
        K, V = wl.kv_tokens(cfg, int(s), int(p.min()), int(p.max() - p.min() + 1), device="cuda")
        idx = torch.as_tensor(p - p.min(), device="cuda")
        Ks.append(K[idx].float().cpu().numpy())
        Vs.append(V[idx].float().cpu().numpy())
    K = np.concatenate(Ks).astype(np.float64)
    V = np.concatenate(Vs).astype(np.float64)
    p64 = run.params64()
    sk = check_codes(oracle, p64, K, kc, kn, cfg.d, run.bits, run.rot)
    sv = check_codes(oracle, p64, V, vc, vn, cfg.d, run.bits, run.rot)
    return {k: sk[k] + sv[k] for k in sk}
