"""Context-parallel decode: the context of every sequence is spread over the ranks of a
process group (one GPU each), each rank holding its slice in its own paged cache.

Softmax attention over disjoint token sets merges exactly by log-sum-exp, the rule the
split-K decode already applies to its chunks ("FreeToken releases", v0.2.0, Kernels:
split decode attention by context length and SM count).  So one decode step is:

1. ``isoq_decode_partial_state`` on this rank's cache: the (acc, m, l) softmax state of
   its slice for every (sequence, query head), in the rotated space;
2. one all-gather of those states over the group (``n_seqs * n_q_heads * (d + 4)``
   floats per rank, e.g. 270 KB for 8 sequences x 64 heads at d = 128);
3. ``isoq_decode_merge_states`` on every rank: merge, normalise, inverse rotation.

Every rank ends with the full output.  The only collective is step 2; the rest runs in
the library's kernels.  RoPE is part of the cached K, so a slice is stored at local
positions 0..n-1 and the ranks' order in the merge does not matter.
"""
from __future__ import annotations

from . import (ISOQ_PAGE_SIZE, Params, PagedCache, isoq_decode_merge_states,
               isoq_decode_partial_state, isoq_decode_state_bytes,
               isoq_decode_workspace_bytes)


def shard_tokens(seq_len: int, world: int, rank: int, page: int = ISOQ_PAGE_SIZE):
    """Token range [start, end) of one sequence that `rank` holds: the pages of the
    context dealt out in contiguous runs whose sizes differ by at most one page."""
    if world < 1 or not 0 <= rank < world or seq_len < 0:
        raise ValueError("bad shard request")
    n_pages = -(-seq_len // page)
    per, extra = divmod(n_pages, world)
    p0 = rank * per + min(rank, extra)
    p1 = p0 + per + (1 if rank < extra else 0)
    return min(p0 * page, seq_len), min(p1 * page, seq_len)


def gather_states(state, group=None):
    """All-gather of the ranks' state tensors: returns [world, *state.shape], entry r =
    rank r's state.  Works on any torch.distributed backend (NCCL over NVLink on GPUs)."""
    import torch.distributed as dist
    if not dist.is_initialized():   # a single-process job holds the whole context
        return state.unsqueeze(0)
    world = dist.get_world_size(group)
    out = state.new_empty((world, *state.shape))
    dist.all_gather(list(out.unbind(0)), state.contiguous(), group=group)
    return out


class CacheSlice:
    """A view of an existing paged cache through another page table (same blocks, same
    status word): e.g. the pages of one rank's slice of each sequence."""

    def __init__(self, cache: PagedCache, page_table):
        from . import isoq_cache
        self.d, self.n_kv_heads, self.n_pages = cache.d, cache.n_kv_heads, cache.n_pages
        self.bits = getattr(cache, "bits", 3)
        self.blocks, self.status = cache.blocks, cache.status
        self.page_table = page_table.to(device=cache.blocks.device,
                                        dtype=page_table.dtype).int().contiguous()
        self._c = isoq_cache(cache.d, cache.n_kv_heads, ISOQ_PAGE_SIZE, cache.n_pages,
                             self.page_table.shape[1], self.page_table.shape[0],
                             cache.blocks.data_ptr(), self.page_table.data_ptr(),
                             cache.status.data_ptr(), self.bits)

    @property
    def c(self):
        return self._c


def slice_of(cache: PagedCache, page_table, lens, world: int, rank: int):
    """This rank's slice of every sequence of a cache that holds whole contexts: a
    CacheSlice over the slice's pages, and the slice lengths."""
    import torch
    pt = page_table.cpu()
    rows, local = [], []
    for s, n in enumerate(lens):
        a, b = shard_tokens(int(n), world, rank)
        rows.append(pt[s, a // ISOQ_PAGE_SIZE:-(-b // ISOQ_PAGE_SIZE)])
        local.append(b - a)
    width = max(1, max(len(r) for r in rows))
    t = torch.zeros((len(rows), width), dtype=torch.int32)
    for s, r in enumerate(rows):
        t[s, :len(r)] = r
    return CacheSlice(cache, t), local


class ContextParallelDecoder:
    """Buffers and calls of one context-parallel decode step on this rank.

    ``cache`` holds this rank's slice of each sequence; ``max_local_len`` bounds the local
    slice lengths (sizes the split plan and the workspace)."""

    def __init__(self, params: Params, cache: PagedCache, n_seqs: int, n_q_heads: int,
                 max_local_len: int, group=None):
        import torch
        self.params, self.cache, self.group = params, cache, group
        self.n_seqs, self.n_q_heads, self.max_local_len = n_seqs, n_q_heads, int(max_local_len)
        d, dev = cache.d, cache.blocks.device
        nb = isoq_decode_workspace_bytes(n_seqs, n_q_heads, cache.n_kv_heads, d, self.max_local_len)
        self.workspace = torch.empty((max(nb, 16),), dtype=torch.uint8, device=dev)
        assert isoq_decode_state_bytes(n_seqs, n_q_heads, d) == n_seqs * n_q_heads * (d + 4) * 4
        self.state = torch.empty((n_seqs, n_q_heads, d + 4), dtype=torch.float32, device=dev)

    def local_state(self, Q, local_lens, scale: float, stream=None):
        isoq_decode_partial_state(self.params, self.cache, Q, local_lens, self.max_local_len,
                                  self.state, scale, self.workspace, stream)
        return self.state

    def __call__(self, Q, local_lens, out, scale: float, stream=None):
        """Q [n_seqs][n_q_heads][d] (same on every rank), local_lens int32 [n_seqs] (this
        rank's slice lengths); writes the attention over the whole contexts to out.

        All three steps run on `stream` (default: the current stream).  The all-gather is
        issued with that stream current, so torch.distributed orders it after the
        partial-state kernel and the merge after the all-gather; a stream other than the
        current one therefore needs no extra synchronisation by the caller."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.state.device)
        with torch.cuda.stream(s):
            self.local_state(Q, local_lens, scale, s)
            states = gather_states(self.state, self.group)
            isoq_decode_merge_states(self.params, states, out, s)
        return out
