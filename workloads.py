"""Seeded synthetic workloads for the packed-KV decode path.

This module draws inputs only: it holds none of the method's arithmetic (no rotation,
no quantisation, no attention).  The same generators feed the CUDA library, the fp64
oracle and the benchmark, so both sides of every parity check see identical inputs.

The pages measure whole-model perplexity and 32K retrieval on real models
("RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused Compressed-Space
Attention", Abstract); neither the weights nor the evaluation data exist here, so these
synthetic K/V/Q tensors stand in for them: heavy tails, per-channel scale spread,
outlier channels and RoPE'd keys imitate real K/V statistics at the pages' 32K scale.

All randomness comes from ``torch.Generator`` objects seeded from (workload, tensor,
sequence, chunk), so any token range of any sequence can be regenerated on its own.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PAGE = 64            # tokens per cache page
CHUNK = 4096         # generation granularity (tokens); a chunk's values depend only on its seed
PARAM_SEED = 0       # rotation-parameter seed used by every workload


@dataclass(frozen=True)
class Workload:
    """One benchmark / parity configuration."""
    idx: int                    # 1-based position in the configuration list
    name: str
    n_seqs: int
    n_q_heads: int
    n_kv_heads: int
    d: int
    kv_dist: str                # "gauss_outlier8" | "student_t4_chscale" | "gauss_outlier10_rope"
                                # | "student_t5" | "gauss_chscale"
    q_dist: str                 # "gauss" | "gauss_outlier8"
    in_dtype: torch.dtype       # K, V and Q element type
    fixed_len: int = 0          # prefill length of every sequence (0: drawn per sequence)
    len_range: tuple = (0, 0)   # inclusive range for drawn lengths
    append_tokens: int = 0      # tokens appended per sequence after the prefill
    quant_chunk: int = 0        # prefill is quantised in calls of this many tokens (0: per seq)
    shuffle_pages: bool = False
    description: str = ""

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def prefill_lens(self) -> list[int]:
        if self.fixed_len:
            return [self.fixed_len] * self.n_seqs
        g = torch.Generator().manual_seed(_seed(self.idx, 8, 0, 0))
        lo, hi = self.len_range
        return torch.randint(lo, hi + 1, (self.n_seqs,), generator=g).tolist()

    def decode_lens(self) -> list[int]:
        return [n + self.append_tokens for n in self.prefill_lens()]


WORKLOADS = [
    Workload(1, "pr1_ref_1k", 1, 8, 2, 128, "gauss_outlier8", "gauss_outlier8", torch.float32,
             fixed_len=1024,
             description="1 sequence, 2 KV heads x 4 query heads (GQA 4), d=128, 1024 tokens; "
                         "K,V,Q fp32 N(0,1) with 4 random channels per head scaled x8; "
                         "quantize all tokens then 1 decode step, scale 1/sqrt(128)"),
    Workload(2, "ctx32k_gqa8", 1, 32, 4, 128, "student_t4_chscale", "gauss", torch.bfloat16,
             fixed_len=32768,
             description="1 sequence, 32 query / 4 KV heads, d=128, 32768 tokens; K,V bf16 "
                         "Student-t(4) x per-channel log-uniform[0.1,10] scales; Q bf16 N(0,1)"),
    Workload(3, "ctx32k_d256_rope", 1, 16, 8, 256, "gauss_outlier10_rope", "gauss",
             torch.bfloat16, fixed_len=32768,
             description="1 sequence, 16 query / 8 KV heads, d=256, 32768 tokens; K,V bf16 "
                         "N(0,1) with 2% of channels x10, RoPE (base 10000) on K"),
    Workload(4, "batched64_paged", 64, 32, 8, 128, "student_t5", "gauss", torch.bfloat16,
             len_range=(4096, 65536), append_tokens=1, shuffle_pages=True,
             description="64 sequences, lengths U{4096..65536}, 32 query / 8 KV heads, d=128, "
                         "64-token pages shuffled in memory; K,V bf16 Student-t(5); append 1 "
                         "token per sequence then decode"),
    Workload(5, "long131k_gqa8", 8, 64, 8, 128, "gauss_chscale", "gauss", torch.bfloat16,
             fixed_len=131072, quant_chunk=16384,
             description="8 sequences x 131072 tokens, 64 query / 8 KV heads (GQA 8), d=128; "
                         "K,V bf16 Gaussian x per-channel log-uniform scales; quantize-append "
                         "in 16384-token chunks, then 1 decode step"),
]


def workload(idx: int) -> Workload:
    return WORKLOADS[idx - 1]


# tensor tags for seed derivation
_K, _V, _Q, _KSCALE, _VSCALE, _KOUT, _VOUT, _LENS, _PERM, _QOUT, _APPK, _APPV = range(1, 13)


def _seed(cfg: int, tag: int, seq: int, chunk: int) -> int:
    return (cfg * 1_000_000_007 + tag * 1_000_003 + seq * 10_007 + chunk * 7 + 12345) % (2**62)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _student_t(shape, nu: int, g, device) -> torch.Tensor:
    """Student-t with integer nu: N(0,1) / sqrt(chi2_nu / nu), chi2 as a sum of squares."""
    z = torch.randn(shape, generator=g, device=device)
    chi2 = torch.zeros(shape, device=device)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=g, device=device) ** 2
    return z / torch.sqrt(chi2 / nu)


def _channel_scales(cfg: Workload, tag: int, device) -> torch.Tensor:
    """[n_kv_heads][d] log-uniform in [0.1, 10]."""
    g = _gen(device, _seed(cfg.idx, tag, 0, 0))
    u = torch.rand((cfg.n_kv_heads, cfg.d), generator=g, device=device)
    return torch.exp(math.log(0.1) + u * (math.log(10.0) - math.log(0.1)))


def _outlier_mult(n_heads: int, d: int, n_ch: int, factor: float, seed: int, device):
    """[n_heads][d] multipliers: n_ch distinct random channels per head get `factor`."""
    g = torch.Generator().manual_seed(seed)
    m = torch.ones((n_heads, d))
    for h in range(n_heads):
        ch = torch.randperm(d, generator=g)[:n_ch]
        m[h, ch] = factor
    return m.to(device)


def _rope_(k: torch.Tensor, pos0: int) -> torch.Tensor:
    """NeoX-style RoPE on [T][H][d] fp32 at positions pos0..pos0+T-1, base 10000, pairing
    (i, i + d/2), theta_i = 10000^(-2i/d)."""
    T, _, d = k.shape
    half = d // 2
    i = torch.arange(half, device=k.device, dtype=torch.float64)
    theta = torch.pow(10000.0, -2.0 * i / d)
    pos = torch.arange(pos0, pos0 + T, device=k.device, dtype=torch.float64)
    ang = pos[:, None] * theta[None, :]
    c = torch.cos(ang).float()[:, None, :]
    s = torch.sin(ang).float()[:, None, :]
    a, b = k[..., :half], k[..., half:]
    return torch.cat([a * c - b * s, a * s + b * c], dim=-1)


def _kv_chunk(cfg: Workload, tag: int, seq: int, chunk: int, device,
              rope: bool = True) -> torch.Tensor:
    """fp32 [CHUNK][n_kv_heads][d] values of K (tag _K) or V (tag _V) for one chunk
    (rope=False: a RoPE workload's keys before the rotary embedding)."""
    g = _gen(device, _seed(cfg.idx, tag, seq, chunk))
    shape = (CHUNK, cfg.n_kv_heads, cfg.d)
    dist = cfg.kv_dist
    if dist == "gauss_outlier8":
        x = torch.randn(shape, generator=g, device=device)
        x *= _outlier_mult(cfg.n_kv_heads, cfg.d, 4, 8.0,
                           _seed(cfg.idx, _KOUT if tag == _K else _VOUT, 0, 0), device)
    elif dist == "student_t4_chscale":
        x = _student_t(shape, 4, g, device)
        x *= _channel_scales(cfg, _KSCALE if tag == _K else _VSCALE, device)
    elif dist == "gauss_outlier10_rope":
        x = torch.randn(shape, generator=g, device=device)
        n_ch = round(0.02 * cfg.d)
        x *= _outlier_mult(cfg.n_kv_heads, cfg.d, n_ch, 10.0,
                           _seed(cfg.idx, _KOUT if tag == _K else _VOUT, 0, 0), device)
        if tag == _K and rope:
            x = _rope_(x, chunk * CHUNK)
    elif dist == "student_t5":
        x = _student_t(shape, 5, g, device)
    elif dist == "gauss_chscale":
        x = torch.randn(shape, generator=g, device=device)
        x *= _channel_scales(cfg, _KSCALE if tag == _K else _VSCALE, device)
    else:
        raise ValueError(dist)
    return x


def kv_tokens(cfg: Workload, seq: int, start: int, count: int, device="cpu", rope: bool = True):
    """K, V of tokens [start, start+count) of sequence `seq`: [count][n_kv_heads][d] in
    cfg.in_dtype.  Any range can be regenerated independently (chunked seeds).  rope=False
    gives a RoPE workload's keys before the rotary embedding (for the fused epilogue)."""
    outs = []
    for tag in (_K, _V):
        parts = []
        c0, c1 = start // CHUNK, (start + count - 1) // CHUNK
        for c in range(c0, c1 + 1):
            x = _kv_chunk(cfg, tag, seq, c, device, rope=rope)
            lo = max(start, c * CHUNK) - c * CHUNK
            hi = min(start + count, (c + 1) * CHUNK) - c * CHUNK
            parts.append(x[lo:hi])
        outs.append(torch.cat(parts).to(cfg.in_dtype).contiguous())
    return outs[0], outs[1]


def queries(cfg: Workload, device="cpu") -> torch.Tensor:
    """Q: [n_seqs][n_q_heads][d] in cfg.in_dtype."""
    g = _gen(device, _seed(cfg.idx, _Q, 0, 0))
    q = torch.randn((cfg.n_seqs, cfg.n_q_heads, cfg.d), generator=g, device=device)
    if cfg.q_dist == "gauss_outlier8":
        q *= _outlier_mult(cfg.n_q_heads, cfg.d, 4, 8.0, _seed(cfg.idx, _QOUT, 0, 0), device)
    return q.to(cfg.in_dtype).contiguous()


def query_chunk(cfg: Workload, n_q: int, device="cpu") -> torch.Tensor:
    """A chunk of n_q query tokens per sequence (chunked prefill / speculative verify):
    [n_seqs][n_q][n_q_heads][d] in cfg.in_dtype, drawn like queries()."""
    g = _gen(device, _seed(cfg.idx, _Q, 1, n_q))
    q = torch.randn((cfg.n_seqs, n_q, cfg.n_q_heads, cfg.d), generator=g, device=device)
    if cfg.q_dist == "gauss_outlier8":
        q *= _outlier_mult(cfg.n_q_heads, cfg.d, 4, 8.0, _seed(cfg.idx, _QOUT, 0, 0), device)
    return q.to(cfg.in_dtype).contiguous()


@dataclass
class PageLayout:
    """Page table of a workload: per sequence, logical page -> physical page id."""
    page_table: torch.Tensor      # int32 [n_seqs][max_pages_per_seq], -1 where unused
    n_pages: int
    capacity: list = field(default_factory=list)   # tokens each sequence can hold


def page_layout(cfg: Workload, extra_tokens: int = 0) -> PageLayout:
    """Allocate ceil((decode_len + extra)/64) pages per sequence; with shuffle_pages the
    physical ids are a seeded random permutation of all pages."""
    caps = [n + extra_tokens for n in cfg.decode_lens()]
    npg = [(c + PAGE - 1) // PAGE for c in caps]
    total = sum(npg)
    if cfg.shuffle_pages:
        g = torch.Generator().manual_seed(_seed(cfg.idx, _PERM, 0, 0))
        ids = torch.randperm(total, generator=g).to(torch.int32)
    else:
        ids = torch.arange(total, dtype=torch.int32)
    maxp = max(npg)
    pt = torch.full((cfg.n_seqs, maxp), -1, dtype=torch.int32)
    o = 0
    for s, n in enumerate(npg):
        pt[s, :n] = ids[o:o + n]
        o += n
    return PageLayout(pt, total, [n * PAGE for n in npg])


def append_kv(cfg: Workload, device="cpu"):
    """The tokens appended after the prefill: K, V [n_seqs * append][n_kv_heads][d] plus the
    int32 seq_ids and positions of each row."""
    lens = cfg.prefill_lens()
    K, V, sid, pos = [], [], [], []
    for s in range(cfg.n_seqs):
        for a in range(cfg.append_tokens):
            g = _gen(device, _seed(cfg.idx, _APPK, s, a))
            k = _kv_like(cfg, g, device, _K, lens[s] + a)
            g = _gen(device, _seed(cfg.idx, _APPV, s, a))
            v = _kv_like(cfg, g, device, _V, lens[s] + a)
            K.append(k)
            V.append(v)
            sid.append(s)
            pos.append(lens[s] + a)
    if not K:
        z = torch.zeros((0, cfg.n_kv_heads, cfg.d), dtype=cfg.in_dtype, device=device)
        e = torch.zeros((0,), dtype=torch.int32, device=device)
        return z, z.clone(), e, e.clone()
    return (torch.cat(K).to(cfg.in_dtype).contiguous(), torch.cat(V).to(cfg.in_dtype).contiguous(),
            torch.tensor(sid, dtype=torch.int32, device=device),
            torch.tensor(pos, dtype=torch.int32, device=device))


def _kv_like(cfg: Workload, g, device, tag: int, position: int) -> torch.Tensor:
    """One appended token [1][n_kv_heads][d] from the same distribution as the prefill."""
    shape = (1, cfg.n_kv_heads, cfg.d)
    if cfg.kv_dist == "student_t5":
        return _student_t(shape, 5, g, device)
    if cfg.kv_dist == "student_t4_chscale":
        return _student_t(shape, 4, g, device) * _channel_scales(
            cfg, _KSCALE if tag == _K else _VSCALE, device)
    if cfg.kv_dist == "gauss_chscale":
        return torch.randn(shape, generator=g, device=device) * _channel_scales(
            cfg, _KSCALE if tag == _K else _VSCALE, device)
    x = torch.randn(shape, generator=g, device=device)
    if cfg.kv_dist == "gauss_outlier8":
        x *= _outlier_mult(cfg.n_kv_heads, cfg.d, 4, 8.0,
                           _seed(cfg.idx, _KOUT if tag == _K else _VOUT, 0, 0), device)
    elif cfg.kv_dist == "gauss_outlier10_rope":
        x *= _outlier_mult(cfg.n_kv_heads, cfg.d, round(0.02 * cfg.d), 10.0,
                           _seed(cfg.idx, _KOUT if tag == _K else _VOUT, 0, 0), device)
        if tag == _K:
            x = _rope_(x, position)
    return x


def prefill_calls(cfg: Workload):
    """The quantize-append calls of the prefill: list of (seq, start, count)."""
    calls = []
    for s, n in enumerate(cfg.prefill_lens()):
        step = cfg.quant_chunk or n
        for a in range(0, n, step):
            calls.append((s, a, min(step, n - a)))
    return calls


def small_variant(cfg: Workload, n_seqs: int | None = None, length: int | None = None,
                  len_range: tuple | None = None) -> Workload:
    """The same distributions at a reduced size (CPU tests and small GPU cases)."""
    from dataclasses import replace
    kw = {}
    if n_seqs is not None:
        kw["n_seqs"] = n_seqs
    if length is not None:
        kw["fixed_len"] = length
        kw["len_range"] = (0, 0)
    if len_range is not None:
        kw["fixed_len"] = 0
        kw["len_range"] = len_range
    if cfg.quant_chunk and length is not None:
        kw["quant_chunk"] = min(cfg.quant_chunk, max(PAGE, length // 2))
    return replace(cfg, **kw)
