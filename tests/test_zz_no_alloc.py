"""The allocation-free decode entry point, isoq_decode_attention_noalloc.

It serves callers that cannot allocate device memory (no allocator of their own to draw a
decode workspace from, or a thread where cudaMalloc may synchronise the device): they pass
only Q, seq_lens and out, and the split-K partial results go to a fixed array inside the
library.  These tests call it through the C ABI and check, on two calls in a row with
different inputs, that it returns what isoq_decode_attention (caller workspace) returns,
bitwise (both run the same split plan and the same kernels, only the partials' address
differs); and that a request larger than the array is refused before anything is
launched.

This file runs last (pytest collects files in name order) and needs nothing from the
other test files, so it passes on its own in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl

pytestmark = pytest.mark.gpu

_fn = iq.raw_lib().isoq_decode_attention_noalloc
_fn.restype = ctypes.c_int
_fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(iq.isoq_cache), ctypes.c_void_p, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                ctypes.c_float, ctypes.c_void_p]


def _case(d, G, lens, seed):
    """A filled paged cache, queries and lengths for one decode call."""
    from dataclasses import replace
    base = wl.workload(1) if d == 128 else wl.workload(3)
    n_kv = 2
    cfg = replace(base, n_seqs=len(lens), n_q_heads=n_kv * G, n_kv_heads=n_kv, d=d,
                  fixed_len=0, len_range=(0, 0))
    params = iq.isoq_make_params(seed, d, n_kv)
    npg = [max(1, -(-n // 64)) for n in lens]
    ids = np.random.default_rng(seed).permutation(sum(npg)).astype(np.int32)
    pt = np.full((len(lens), max(npg)), -1, np.int32)
    o = 0
    for s, n in enumerate(npg):
        pt[s, :n] = ids[o:o + n]
        o += n
    cache = iq.PagedCache(d, n_kv, int(sum(npg)), torch.from_numpy(pt))
    for s, n in enumerate(lens):
        K, V = wl.kv_tokens(cfg, s, 0, n, device="cuda")
        iq.isoq_quantize_append(params, cache, K, V,
                                torch.full((n,), s, dtype=torch.int32, device="cuda"),
                                torch.arange(n, dtype=torch.int32, device="cuda"))
    Q = wl.queries(cfg, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return cfg, params, cache, Q, sl


def _with_workspace(cfg, params, cache, Q, sl, max_len):
    out = torch.empty((Q.shape[0], Q.shape[1], cfg.d), dtype=torch.float32, device="cuda")
    nb = iq.isoq_decode_workspace_bytes(Q.shape[0], Q.shape[1], cfg.n_kv_heads, cfg.d, max_len)
    ws = torch.empty((nb,), dtype=torch.uint8, device="cuda")
    iq.isoq_decode_attention(params, cache, Q, sl, max_len, out, cfg.scale, ws)
    return out


def _noalloc(cfg, params, cache, Q, sl, max_len):
    out = torch.full((Q.shape[0], Q.shape[1], cfg.d), float("nan"), dtype=torch.float32,
                     device="cuda")
    rc = _fn(params.handle, ctypes.byref(cache.c), Q.data_ptr(), iq._dtype_code(Q), Q.shape[0],
             Q.shape[1], sl.data_ptr(), max_len, out.data_ptr(), cfg.scale,
             torch.cuda.current_stream().cuda_stream)
    assert rc == iq.ISOQ_OK, iq.isoq_error_string(rc)
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cases = [(128, 4, [1000, 3000, 65], 11), (256, 8, [2049, 7], 12)]
    for d, G, lens, seed in cases:          # two calls in a row, different shapes and data
        cfg, params, cache, Q, sl = _case(d, G, lens, seed)
        max_len = max(lens) + 500          # leaves some splits empty
        ref = _with_workspace(cfg, params, cache, Q, sl, max_len)
        got = _noalloc(cfg, params, cache, Q, sl, max_len)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref)        # same plan, same kernels: identical results
        assert iq.isoq_get_status(cache) == 0
    assert iq.isoq_last_cuda_error() == 0


def test_noalloc_rejects_requests_larger_than_its_array():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d, n_kv, G = 256, 8, 16
    n_seqs = 64   # more sequences until one decode's partials exceed the array
    while iq.isoq_decode_workspace_bytes(n_seqs, n_kv * G, n_kv, d, 4096) <= \
            iq.ISOQ_NOALLOC_SCRATCH_BYTES:
        n_seqs *= 2
    params = iq.isoq_make_params(0, d, n_kv)
    cache = iq.PagedCache(d, n_kv, 1, torch.zeros((n_seqs, 1), dtype=torch.int32))
    need = iq.isoq_decode_workspace_bytes(n_seqs, n_kv * G, n_kv, d, 4096)
    assert need > iq.ISOQ_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros((n_seqs, n_kv * G, d), dtype=torch.float32, device="cuda")
    sl = torch.zeros((n_seqs,), dtype=torch.int32, device="cuda")
    before = dummy.clone()
    rc = _fn(params.handle, ctypes.byref(cache.c), dummy.data_ptr(), iq.ISOQ_F32, n_seqs,
             n_kv * G, sl.data_ptr(), 4096, dummy.data_ptr(), 0.1, None)
    assert rc == iq.ISOQ_E_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(dummy, before)       # nothing was launched
