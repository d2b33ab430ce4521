"""Python binding of libisoq (IsoQuant 3-bit KV cache + decode attention on the packed
cache, CUDA for sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch supplies device memory and streams.  The functions carry the C names of
``include/isoq.h`` and raise :class:`IsoqError` on a negative return code.  Importing
this package fails loudly if ``libisoq.so`` has not been built
(``python rotated_bit_kv_isoquant_b200/build.py``); there is no fallback.

With ``ISOQ_CHECK_BOUNDS=1`` in the environment at import, the package loads the
bounds-checked build ``libisoq_checked.so`` (``build.py --checked``) instead: the same
entry points, every kernel index compared with its extent, ISOQ_ST_BOUNDS set in the
status word where one is not.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("ISOQ_CHECK_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libisoq_checked.so" if CHECKED else "libisoq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{os.path.basename(LIB_PATH)} is missing at {LIB_PATH}: build it with "
        "`python rotated_bit_kv_isoquant_b200/build.py" + (" --checked" if CHECKED else "") +
        "` (nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

ISOQ_OK = 0
ISOQ_E_ARG = -1
ISOQ_E_DIM = -2
ISOQ_E_GQA = -3
ISOQ_E_WORKSPACE = -4
ISOQ_E_CUDA = -5
ISOQ_E_DEVICE = -6

ISOQ_ST_SEQ_RANGE = 0x1
ISOQ_ST_POS_RANGE = 0x2
ISOQ_ST_PAGE_RANGE = 0x4
ISOQ_ST_NORM_SAT = 0x8
ISOQ_ST_LEN_RANGE = 0x10
ISOQ_ST_TIMEOUT = 0x20
ISOQ_ST_BOUNDS = 0x40

ISOQ_F32, ISOQ_BF16, ISOQ_F16 = 0, 1, 2
ISOQ_ROT_SO4, ISOQ_ROT_SO2 = 0, 1
ISOQ_PAGE_SIZE = 64
ISOQ_NOALLOC_SCRATCH_BYTES = 16 << 20


class IsoqError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _lib.isoq_error_string(code).decode()
        if code == ISOQ_E_CUDA:
            msg += f" (cudaError {_lib.isoq_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [{code}]")
        self.code = code


class isoq_cache(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("page_size", ctypes.c_int),
                ("n_pages", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int),
                ("n_seqs", ctypes.c_int), ("blocks", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("status", ctypes.c_void_p),
                ("bits", ctypes.c_int)]


_p, _i, _sz, _u64, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_float
_cp = ctypes.POINTER(isoq_cache)

_SIGS = {
    "isoq_params_generate": (_i, [_u64, _i, _i, _p]),
    "isoq_params_generate_v": (_i, [_u64, _i, _i, _i, _p]),
    "isoq_make_params_v": (_i, [_u64, _i, _i, _i, _i, ctypes.POINTER(_p)]),
    "isoq_params_format": (_i, [_p, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "isoq_block_bytes_v": (_sz, [_i, _i, _i]),
    "isoq_make_params": (_i, [_u64, _i, _i, ctypes.POINTER(_p)]),
    "isoq_params_copy": (_i, [_p, _p]),
    "isoq_params_shape": (_i, [_p, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "isoq_params_destroy": (None, [_p]),
    "isoq_block_bytes": (_sz, [_i, _i]),
    "isoq_quantize_append": (_i, [_p, _cp, _p, _p, _i, _i, _p, _p, _p]),
    "isoq_quantize_append_rope": (_i, [_p, _cp, _p, _p, _i, _i, _p, _p, _p, _i, _p]),
    "isoq_quantize_append_layers": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p, _p, _i, _p]),
    "isoq_rope_table_bytes": (_sz, [_i, _i]),
    "isoq_rope_table": (_i, [_p, _i, _i, ctypes.c_double, _p]),
    "isoq_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "isoq_decode_num_splits": (_i, [_i, _i, _i, _i, _i]),
    "isoq_decode_attention": (_i, [_p, _cp, _p, _i, _i, _i, _p, _i, _p, _f, _p, _sz, _p]),
    "isoq_decode_attention_noalloc": (_i, [_p, _cp, _p, _i, _i, _i, _p, _i, _p, _f, _p]),
    "isoq_decode_state_bytes": (_sz, [_i, _i, _i]),
    "isoq_multi_token_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "isoq_multi_token_attention": (_i, [_p, _cp, _p, _i, _i, _i, _i, _p, _i, _p, _f, _p, _sz, _p]),
    "isoq_decode_partial_state": (_i, [_p, _cp, _p, _i, _i, _i, _p, _i, _p, _f, _p, _sz, _p]),
    "isoq_decode_merge_states": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "isoq_get_status": (_i, [_cp, ctypes.POINTER(ctypes.c_uint32)]),
    "isoq_reset_status": (_i, [_cp, _p]),
    "isoq_last_cuda_error": (_i, []),
    "isoq_selftest_bounded_wait": (_i, [_p, ctypes.c_uint, _p, _p]),
    "isoq_selftest_bounds": (_i, [_p, _p]),
    "isoq_error_string": (ctypes.c_char_p, [_i]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def _check(rc: int, where: str):
    if rc < 0:
        raise IsoqError(rc, where)
    return rc


def _dtype_code(t) -> int:
    import torch
    m = {torch.float32: ISOQ_F32, torch.bfloat16: ISOQ_BF16, torch.float16: ISOQ_F16}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _dev_ptr(t, name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ------------------------------------------------------------------------------------
# Parameters
# ------------------------------------------------------------------------------------
def _params_shape(d: int, n_kv_heads: int, rotation: int):
    return (n_kv_heads, d // 2, 2) if rotation == ISOQ_ROT_SO2 else (n_kv_heads, d // 4, 2, 4)


def isoq_params_generate(seed: int, d: int, n_kv_heads: int,
                         rotation: int = ISOQ_ROT_SO4) -> np.ndarray:
    """Host-side rotation parameters, float32 [n_kv_heads][d/4][2][4] (SO(4) quaternion
    pairs) or [n_kv_heads][d/2][2] (SO(2) cos, sin); no GPU needed."""
    out = np.zeros(_params_shape(d, n_kv_heads, rotation), dtype=np.float32)
    _check(_lib.isoq_params_generate_v(seed, d, n_kv_heads, rotation, out.ctypes.data),
           "isoq_params_generate_v")
    return out


class Params:
    """Owning wrapper of an ``isoq_params*`` handle."""

    def __init__(self, handle: int, d: int, n_kv_heads: int, bits: int = 3,
                 rotation: int = ISOQ_ROT_SO4):
        self.handle = handle
        self.d = d
        self.n_kv_heads = n_kv_heads
        self.bits = bits
        self.rotation = rotation

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.isoq_params_destroy(h)


def isoq_make_params(seed: int, d: int, n_kv_heads: int, bits: int = 3,
                     rotation: int = ISOQ_ROT_SO4) -> Params:
    """Parameters of the method (3 bits, SO(4) blocks) or of a format variant."""
    h = _p()
    _check(_lib.isoq_make_params_v(seed, d, n_kv_heads, bits, rotation, ctypes.byref(h)),
           "isoq_make_params_v")
    return Params(h.value, d, n_kv_heads, bits, rotation)


def isoq_params_format(params: Params):
    b, r = _i(), _i()
    _check(_lib.isoq_params_format(params.handle, ctypes.byref(b), ctypes.byref(r)),
           "isoq_params_format")
    return b.value, r.value


def isoq_params_copy(params: Params) -> np.ndarray:
    out = np.zeros(_params_shape(params.d, params.n_kv_heads, params.rotation), dtype=np.float32)
    _check(_lib.isoq_params_copy(params.handle, out.ctypes.data), "isoq_params_copy")
    return out


def isoq_params_shape(params: Params):
    d, h = _i(), _i()
    _check(_lib.isoq_params_shape(params.handle, ctypes.byref(d), ctypes.byref(h)),
           "isoq_params_shape")
    return d.value, h.value


def isoq_params_destroy(params: Params) -> None:
    h, params.handle = params.handle, None
    if h:
        _lib.isoq_params_destroy(h)


# ------------------------------------------------------------------------------------
# Cache
# ------------------------------------------------------------------------------------
def isoq_block_bytes(d: int, page_size: int = ISOQ_PAGE_SIZE, bits: int = 3) -> int:
    return int(_lib.isoq_block_bytes_v(d, bits, page_size))


class PagedCache:
    """Device memory of a paged cache (torch tensors) plus its ``isoq_cache`` view."""

    def __init__(self, d: int, n_kv_heads: int, n_pages: int, page_table, device=None,
                 bits: int = 3):
        import torch
        device = device or torch.device("cuda")
        self.d, self.n_kv_heads, self.n_pages, self.bits = d, n_kv_heads, n_pages, bits
        bb = isoq_block_bytes(d, bits=bits)
        if bb == 0:
            raise IsoqError(ISOQ_E_DIM, "PagedCache")
        self.blocks = torch.zeros((n_pages, n_kv_heads, bb), dtype=torch.uint8, device=device)
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        self._c = isoq_cache(d, n_kv_heads, ISOQ_PAGE_SIZE, n_pages, self.page_table.shape[1],
                             self.page_table.shape[0], self.blocks.data_ptr(),
                             self.page_table.data_ptr(), self.status.data_ptr(), bits)

    @property
    def c(self) -> isoq_cache:
        return self._c


# ------------------------------------------------------------------------------------
# Kernels
# ------------------------------------------------------------------------------------
def isoq_quantize_append(params: Params, cache: PagedCache, K, V, seq_ids, positions,
                         stream=None) -> None:
    """K, V: CUDA [n_tokens][n_kv_heads][d] (fp32/bf16/fp16); seq_ids, positions: int32."""
    import torch
    if K.dtype != V.dtype or K.shape != V.shape:
        raise ValueError("K and V must have the same shape and dtype")
    n = K.shape[0]
    _check(_lib.isoq_quantize_append(
        params.handle, ctypes.byref(cache.c), _dev_ptr(K, "K"), _dev_ptr(V, "V"), _dtype_code(K),
        n, _dev_ptr(seq_ids, "seq_ids", torch.int32), _dev_ptr(positions, "positions", torch.int32),
        _stream_ptr(stream)), "isoq_quantize_append")


def isoq_rope_table(d: int, max_pos: int, base: float = 10000.0, device=None, stream=None):
    """Device fp32 [max_pos][d/2][2] table of (cos, sin)(pos * base^(-2i/d)), computed in
    fp64 on the GPU, for the fused RoPE quantize-append."""
    import torch
    nbytes = int(_lib.isoq_rope_table_bytes(d, max_pos))
    if nbytes == 0:
        raise IsoqError(ISOQ_E_DIM, "isoq_rope_table")
    t = torch.empty((max_pos, d // 2, 2), dtype=torch.float32, device=device or "cuda")
    _check(_lib.isoq_rope_table(t.data_ptr(), d, max_pos, float(base), _stream_ptr(stream)),
           "isoq_rope_table")
    return t


def isoq_quantize_append_rope(params: Params, cache: PagedCache, K, V, seq_ids, positions,
                              rope_table, stream=None) -> None:
    """isoq_quantize_append with the rotary embedding applied to K (pre-RoPE keys) at each
    token's position, from rope_table (isoq_rope_table)."""
    import torch
    if K.dtype != V.dtype or K.shape != V.shape:
        raise ValueError("K and V must have the same shape and dtype")
    _check(_lib.isoq_quantize_append_rope(
        params.handle, ctypes.byref(cache.c), _dev_ptr(K, "K"), _dev_ptr(V, "V"), _dtype_code(K),
        K.shape[0], _dev_ptr(seq_ids, "seq_ids", torch.int32),
        _dev_ptr(positions, "positions", torch.int32),
        _dev_ptr(rope_table, "rope_table", torch.float32), rope_table.shape[0],
        _stream_ptr(stream)), "isoq_quantize_append_rope")


def isoq_quantize_append_layers(params_list, caches, Ks, Vs, seq_ids, positions,
                                rope_table=None, stream=None) -> None:
    """One quantize-append of the same tokens into several layers' caches (one launch per
    up to 32 layers): params_list, caches, Ks, Vs are per-layer sequences."""
    import torch
    n = len(params_list)
    if not (n == len(caches) == len(Ks) == len(Vs)) or n == 0:
        raise ValueError("one params, cache, K and V per layer")
    if any(t.dtype != Ks[0].dtype or t.shape != Ks[0].shape for t in list(Ks) + list(Vs)):
        raise ValueError("every layer's K and V must have the same shape and dtype")
    P = (_p * n)(*[p.handle for p in params_list])
    C = (_p * n)(*[ctypes.addressof(c.c) for c in caches])
    Kp = (_p * n)(*[_dev_ptr(k, "K") for k in Ks])
    Vp = (_p * n)(*[_dev_ptr(v, "V") for v in Vs])
    _check(_lib.isoq_quantize_append_layers(
        P, C, Kp, Vp, n, _dtype_code(Ks[0]), Ks[0].shape[0],
        _dev_ptr(seq_ids, "seq_ids", torch.int32), _dev_ptr(positions, "positions", torch.int32),
        _dev_ptr(rope_table, "rope_table", torch.float32) if rope_table is not None else None,
        rope_table.shape[0] if rope_table is not None else 0, _stream_ptr(stream)),
        "isoq_quantize_append_layers")


def isoq_decode_workspace_bytes(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len) -> int:
    return int(_lib.isoq_decode_workspace_bytes(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len))


def isoq_decode_num_splits(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len) -> int:
    return _check(_lib.isoq_decode_num_splits(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len),
                  "isoq_decode_num_splits")


def isoq_decode_attention(params: Params, cache: PagedCache, Q, seq_lens, max_seq_len: int,
                          out, scale: float, workspace, stream=None) -> None:
    """Q: CUDA [n_seqs][n_q_heads][d]; seq_lens int32 [n_seqs]; out fp32 like Q;
    workspace: CUDA uint8 tensor of >= isoq_decode_workspace_bytes(...) bytes."""
    import torch
    n_seqs, n_q_heads = Q.shape[0], Q.shape[1]
    _check(_lib.isoq_decode_attention(
        params.handle, ctypes.byref(cache.c), _dev_ptr(Q, "Q"), _dtype_code(Q), n_seqs, n_q_heads,
        _dev_ptr(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _dev_ptr(out, "out", torch.float32), float(scale), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
        "isoq_decode_attention")


def isoq_decode_attention_noalloc(params: Params, cache: PagedCache, Q, seq_lens,
                                  max_seq_len: int, out, scale: float, stream=None) -> None:
    """isoq_decode_attention without a workspace, for callers that cannot allocate device
    memory: the partial results use a fixed 16 MiB array inside the library (one per GPU,
    shared by all calls, so calls must not overlap on the GPU)."""
    import torch
    _check(_lib.isoq_decode_attention_noalloc(
        params.handle, ctypes.byref(cache.c), _dev_ptr(Q, "Q"), _dtype_code(Q), Q.shape[0],
        Q.shape[1], _dev_ptr(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _dev_ptr(out, "out", torch.float32), float(scale), _stream_ptr(stream)),
        "isoq_decode_attention_noalloc")


def isoq_multi_token_workspace_bytes(n_seqs, n_q, n_q_heads, n_kv_heads, d, max_seq_len) -> int:
    return int(_lib.isoq_multi_token_workspace_bytes(n_seqs, n_q, n_q_heads, n_kv_heads, d,
                                                     max_seq_len))


def isoq_multi_token_attention(params: Params, cache: PagedCache, Q, seq_lens, max_seq_len: int,
                               out, scale: float, workspace, stream=None) -> None:
    """Causal attention of a chunk of query tokens per sequence on the packed cache.
    Q: CUDA [n_seqs][n_q][n_q_heads][d] (query i at position seq_len - n_q + i); out fp32
    like Q; workspace >= isoq_multi_token_workspace_bytes(...) bytes."""
    import torch
    n_seqs, n_q, n_q_heads = Q.shape[0], Q.shape[1], Q.shape[2]
    _check(_lib.isoq_multi_token_attention(
        params.handle, ctypes.byref(cache.c), _dev_ptr(Q, "Q"), _dtype_code(Q), n_seqs, n_q,
        n_q_heads, _dev_ptr(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _dev_ptr(out, "out", torch.float32), float(scale), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
        "isoq_multi_token_attention")


def isoq_decode_state_bytes(n_seqs, n_q_heads, d) -> int:
    return int(_lib.isoq_decode_state_bytes(n_seqs, n_q_heads, d))


def isoq_decode_partial_state(params: Params, cache: PagedCache, Q, seq_lens, max_seq_len: int,
                              state, scale: float, workspace, stream=None) -> None:
    """Softmax state of this cache's slice of every context: state fp32 CUDA
    [n_seqs][n_q_heads][d + 4] = (acc[d], m, l, 0, 0); other arguments as
    isoq_decode_attention."""
    import torch
    n_seqs, n_q_heads = Q.shape[0], Q.shape[1]
    _check(_lib.isoq_decode_partial_state(
        params.handle, ctypes.byref(cache.c), _dev_ptr(Q, "Q"), _dtype_code(Q), n_seqs, n_q_heads,
        _dev_ptr(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _dev_ptr(state, "state", torch.float32), float(scale), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
        "isoq_decode_partial_state")


def isoq_decode_merge_states(params: Params, states, out, stream=None) -> None:
    """states: fp32 CUDA [n_states][n_seqs][n_q_heads][d + 4] (gathered slice states);
    out: fp32 CUDA [n_seqs][n_q_heads][d], attention over the union of the slices."""
    import torch
    n_states, n_seqs, n_q_heads = states.shape[0], states.shape[1], states.shape[2]
    _check(_lib.isoq_decode_merge_states(
        params.handle, _dev_ptr(states, "states", torch.float32), n_states, n_seqs, n_q_heads,
        _dev_ptr(out, "out", torch.float32), _stream_ptr(stream)), "isoq_decode_merge_states")


def isoq_get_status(cache: PagedCache) -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.isoq_get_status(ctypes.byref(cache.c), ctypes.byref(v)), "isoq_get_status")
    return int(v.value)


def isoq_reset_status(cache: PagedCache, stream=None) -> None:
    _check(_lib.isoq_reset_status(ctypes.byref(cache.c), _stream_ptr(stream)), "isoq_reset_status")


def isoq_last_cuda_error() -> int:
    return int(_lib.isoq_last_cuda_error())


def isoq_selftest_bounded_wait(polls: int = 4096, stream=None):
    """Runs the bounded-wait self-test; returns (status word, stuck wait gave up, completed
    wait succeeded)."""
    import torch
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    result = torch.zeros((2,), dtype=torch.int32, device="cuda")
    _check(_lib.isoq_selftest_bounded_wait(status.data_ptr(), polls, result.data_ptr(),
                                           _stream_ptr(stream)), "isoq_selftest_bounded_wait")
    torch.cuda.synchronize()
    r = result.cpu().tolist()
    return int(status.item()) & 0xffffffff, bool(r[0]), bool(r[1])


def isoq_selftest_bounds(stream=None) -> int:
    """Runs the bounds-check self-test (one index equal to its extent); returns the status
    word: ISOQ_ST_BOUNDS set by the checked build, clear in the normal one."""
    import torch
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    _check(_lib.isoq_selftest_bounds(status.data_ptr(), _stream_ptr(stream)),
           "isoq_selftest_bounds")
    torch.cuda.synchronize()
    return int(status.item()) & 0xffffffff


def isoq_error_string(code: int) -> str:
    return _lib.isoq_error_string(code).decode()


def raw_lib() -> ctypes.CDLL:
    """The loaded ctypes library (for raw C-ABI calls)."""
    return _lib
