"""IsoQuant fp64 CPU oracle: ctypes shim over ``isoq_oracle.c``.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package.  It shares no code
with the CUDA library and never imports the product package.

Every function follows the method page "RotaryQuant: Fitting 120B MoE Models on Consumer
Hardware via Fused Compressed-Space Attention", Abstract (WHT, block-diagonal SO(4)
rotations, 3-bit scalar quantisation, attention on the packed tensors); the readings the
pages leave open are listed at the top of ``isoq_oracle.c``.  All arithmetic is fp64.

Variants of the same family take ``bits`` (2, 3 or 4: the Lloyd-Max codebook size) and
``rot`` (0: SO(4) quaternion blocks, IsoQuant; 1: SO(2) blocks, the PlanarQuant variant the
same abstract names); the defaults are the method's 3 bits and SO(4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "isoq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libisoq_oracle.so")

_GCC_FLAGS = ["-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
              "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_d = ctypes.c_double
_i = ctypes.c_int
_p = ctypes.c_void_p


def _declare(L):
    L.ref_level.restype = _d
    L.ref_level.argtypes = [_i]
    L.ref_threshold.restype = _d
    L.ref_threshold.argtypes = [_i]
    L.ref_num_threads.restype = _i
    L.ref_set_num_threads.restype = None
    L.ref_set_num_threads.argtypes = [_i]
    L.ref_splitmix64_next.restype = ctypes.c_uint64
    L.ref_splitmix64_next.argtypes = [_p]
    L.ref_normal.restype = _d
    L.ref_normal.argtypes = [_p]
    L.ref_make_params.restype = None
    L.ref_make_params.argtypes = [ctypes.c_uint64, _i, _i, _p, _p]
    L.ref_wht.restype = None
    L.ref_wht.argtypes = [_p, _i]
    L.ref_quat_mul.restype = None
    L.ref_quat_mul.argtypes = [_p, _p, _p]
    L.ref_so4_forward.restype = None
    L.ref_so4_forward.argtypes = [_p, _p, _p, _p]
    L.ref_so4_inverse.restype = None
    L.ref_so4_inverse.argtypes = [_p, _p, _p, _p]
    L.ref_rotate.restype = None
    L.ref_rotate.argtypes = [_p, _p, _p, _i]
    L.ref_unrotate.restype = None
    L.ref_unrotate.argtypes = [_p, _p, _p, _i]
    L.ref_fp16_bits.restype = ctypes.c_uint16
    L.ref_fp16_bits.argtypes = [_d]
    L.ref_fp16_value.restype = _d
    L.ref_fp16_value.argtypes = [ctypes.c_uint16]
    L.ref_quantize_vector.restype = _i
    L.ref_quantize_vector.argtypes = [_p, _p, _i, _p, _p, _p]
    L.ref_pack_codes.restype = None
    L.ref_pack_codes.argtypes = [_p, _i, _p]
    L.ref_unpack_codes.restype = None
    L.ref_unpack_codes.argtypes = [_p, _i, _p]
    L.ref_block_bytes.restype = ctypes.c_size_t
    L.ref_block_bytes.argtypes = [_i, _i]
    L.ref_quantize_append.restype = _i
    L.ref_quantize_append.argtypes = [_p, _i, _i, _i, _p, _p, _i, _p, _p, _i, _p, _p]
    L.ref_dequantize_slot.restype = None
    L.ref_dequantize_slot.argtypes = [_p, _i, _i, _i, _p, _i, _i, _i, _i, _p]
    L.ref_decode_attention.restype = None
    L.ref_decode_attention.argtypes = [_p, _i, _i, _i, _p, _p, _i, _i, _i, _p, _p, _d, _p,
                                       _p, _i]
    L.ref_quantize_rows.restype = None
    L.ref_quantize_rows.argtypes = [_p, _i, _i, _p, _i, _p, _p, _p]
    L.ref_unpack_codes_batch.restype = None
    L.ref_unpack_codes_batch.argtypes = [_p, _i, ctypes.c_long, _p]
    L.ref_attention_full.restype = None
    L.ref_attention_full.argtypes = [_i, _i, _i, _i, _p, _p, _p, _d, _p]
    L.ref_rope.restype = None
    L.ref_rope.argtypes = [_p, _i, _i, _d, _p]
    L.ref_level_v.restype = _d
    L.ref_level_v.argtypes = [_i, _i]
    L.ref_threshold_v.restype = _d
    L.ref_threshold_v.argtypes = [_i, _i]
    L.ref_make_params_so2.restype = None
    L.ref_make_params_so2.argtypes = [ctypes.c_uint64, _i, _i, _p, _p]
    L.ref_params_per_head.restype = _i
    L.ref_params_per_head.argtypes = [_i, _i]
    L.ref_so2_forward.restype = None
    L.ref_so2_forward.argtypes = [_p, _p, _p]
    L.ref_so2_inverse.restype = None
    L.ref_so2_inverse.argtypes = [_p, _p, _p]
    L.ref_rotate_v.restype = None
    L.ref_rotate_v.argtypes = [_i, _p, _p, _p, _i]
    L.ref_unrotate_v.restype = None
    L.ref_unrotate_v.argtypes = [_i, _p, _p, _p, _i]
    L.ref_quantize_vector_v.restype = _i
    L.ref_quantize_vector_v.argtypes = [_i, _i, _p, _p, _i, _p, _p, _p]
    L.ref_pack_codes_v.restype = None
    L.ref_pack_codes_v.argtypes = [_i, _p, _i, _p]
    L.ref_unpack_codes_v.restype = None
    L.ref_unpack_codes_v.argtypes = [_i, _p, _i, _p]
    L.ref_block_bytes_v.restype = ctypes.c_size_t
    L.ref_block_bytes_v.argtypes = [_i, _i, _i]
    L.ref_quantize_append_v.restype = _i
    L.ref_quantize_append_v.argtypes = [_i, _i, _p, _i, _i, _i, _p, _p, _i, _p, _p, _i, _p, _p]
    L.ref_dequantize_slot_v.restype = None
    L.ref_dequantize_slot_v.argtypes = [_i, _i, _p, _i, _i, _i, _p, _i, _i, _i, _i, _p]
    L.ref_decode_attention_v.restype = None
    L.ref_decode_attention_v.argtypes = [_i, _i, _p, _i, _i, _i, _p, _p, _i, _i, _i, _p, _p, _d,
                                         _p, _p, _i]
    L.ref_quantize_rows_v.restype = None
    L.ref_quantize_rows_v.argtypes = [_i, _i, _p, _i, _i, _p, _i, _p, _p, _p]
    L.ref_unpack_codes_batch_v.restype = None
    L.ref_unpack_codes_batch_v.argtypes = [_i, _p, _i, ctypes.c_long, _p]
    L.ref_v_put_codes.restype = None
    L.ref_v_put_codes.argtypes = [_i, _i, _i, _p, _i, _p]
    L.ref_v_get_codes.restype = None
    L.ref_v_get_codes.argtypes = [_i, _i, _i, _p, _i, _p]
    L.ref_v_region_records.restype = None
    L.ref_v_region_records.argtypes = [_i, _i, _i, _p, _p]


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


# ------------------------------------------------------------------------------------
# Constants
# ------------------------------------------------------------------------------------
def levels(bits: int = 3) -> np.ndarray:
    """The 2^bits codebook levels in N(0,1) units, ascending (Lloyd-Max, Max 1960)."""
    return np.array([lib().ref_level_v(bits, c) for c in range(1 << bits)])


def thresholds(bits: int = 3) -> np.ndarray:
    """The 2^bits - 1 decision thresholds: midpoints of adjacent levels."""
    return np.array([lib().ref_threshold_v(bits, j) for j in range((1 << bits) - 1)])


def num_threads() -> int:
    return int(lib().ref_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops from now on (timing only)."""
    lib().ref_set_num_threads(int(n))


# ------------------------------------------------------------------------------------
# Parameters and rotations
# ------------------------------------------------------------------------------------
def splitmix64_stream(seed: int, n: int) -> np.ndarray:
    st = ctypes.c_uint64(seed)
    return np.array([lib().ref_splitmix64_next(ctypes.byref(st)) for _ in range(n)],
                    dtype=np.uint64)


def normals(seed: int, n: int) -> np.ndarray:
    st = ctypes.c_uint64(seed)
    return np.array([lib().ref_normal(ctypes.byref(st)) for _ in range(n)])


def make_params(seed: int, d: int, n_kv_heads: int):
    """(params64, params32), each [n_kv_heads][d/4][2][4]: per block p then q (w,x,y,z)."""
    p64 = np.zeros((n_kv_heads, d // 4, 2, 4), dtype=np.float64)
    p32 = np.zeros((n_kv_heads, d // 4, 2, 4), dtype=np.float32)
    lib().ref_make_params(ctypes.c_uint64(seed), d, n_kv_heads, _ptr(p64), _ptr(p32))
    return p64, p32


def make_params_so2(seed: int, d: int, n_kv_heads: int):
    """(params64, params32), each [n_kv_heads][d/2][2]: per 2x2 block (cos phi, sin phi)."""
    p64 = np.zeros((n_kv_heads, d // 2, 2), dtype=np.float64)
    p32 = np.zeros((n_kv_heads, d // 2, 2), dtype=np.float32)
    lib().ref_make_params_so2(ctypes.c_uint64(seed), d, n_kv_heads, _ptr(p64), _ptr(p32))
    return p64, p32


def make_params_v(seed: int, d: int, n_kv_heads: int, rot: int = 0):
    """make_params (rot 0, SO(4)) or make_params_so2 (rot 1)."""
    return make_params_so2(seed, d, n_kv_heads) if rot == 1 else make_params(seed, d, n_kv_heads)


def so2_forward(cs, y) -> np.ndarray:
    cs, y = _f64(cs), _f64(y)
    z = np.zeros(2)
    lib().ref_so2_forward(_ptr(cs), _ptr(y), _ptr(z))
    return z


def so2_inverse(cs, z) -> np.ndarray:
    cs, z = _f64(cs), _f64(z)
    y = np.zeros(2)
    lib().ref_so2_inverse(_ptr(cs), _ptr(z), _ptr(y))
    return y


def wht(x) -> np.ndarray:
    """Orthonormal natural-order WHT of each row of x (last axis = d)."""
    x = _f64(x).copy()
    flat = x.reshape(-1, x.shape[-1])
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib().ref_wht(_ptr(row), row.shape[0])
        flat[r] = row
    return flat.reshape(x.shape)


def quat_mul(a, b) -> np.ndarray:
    a, b = _f64(a), _f64(b)
    out = np.zeros(4)
    lib().ref_quat_mul(_ptr(a), _ptr(b), _ptr(out))
    return out


def so4_forward(p, q, y) -> np.ndarray:
    p, q, y = _f64(p), _f64(q), _f64(y)
    z = np.zeros(4)
    lib().ref_so4_forward(_ptr(p), _ptr(q), _ptr(y), _ptr(z))
    return z


def so4_inverse(p, q, z) -> np.ndarray:
    p, q, z = _f64(p), _f64(q), _f64(z)
    y = np.zeros(4)
    lib().ref_so4_inverse(_ptr(p), _ptr(q), _ptr(z), _ptr(y))
    return y


def rotate(params_head, x, rot: int = 0) -> np.ndarray:
    """z = R x for one head: WHT then the blocks (rot 0: SO(4), params_head [d/4][2][4];
    rot 1: SO(2), params_head [d/2][2])."""
    ph, x = _f64(params_head), _f64(x)
    z = np.zeros_like(x)
    lib().ref_rotate_v(rot, _ptr(ph), _ptr(x), _ptr(z), x.shape[-1])
    return z


def unrotate(params_head, z, rot: int = 0) -> np.ndarray:
    ph, z = _f64(params_head), _f64(z)
    x = np.zeros_like(z)
    lib().ref_unrotate_v(rot, _ptr(ph), _ptr(z), _ptr(x), z.shape[-1])
    return x


def rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of each row of x (last axis d) at positions pos (scalar or one per
    row): dims (i, i + d/2) rotated by pos * base^(-2i/d)."""
    x = _f64(x)
    flat = x.reshape(-1, x.shape[-1])
    pos = np.broadcast_to(np.asarray(pos, dtype=np.int64), (flat.shape[0],))
    out = np.zeros_like(flat)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        o = np.zeros_like(row)
        lib().ref_rope(_ptr(row), row.shape[0], int(pos[r]), float(base), _ptr(o))
        out[r] = o
    return out.reshape(x.shape)


# ------------------------------------------------------------------------------------
# binary16
# ------------------------------------------------------------------------------------
def fp16_bits(v: float) -> int:
    return int(lib().ref_fp16_bits(float(v)))


def fp16_value(h: int) -> float:
    return float(lib().ref_fp16_value(int(h)))


# ------------------------------------------------------------------------------------
# Quantisation and packing
# ------------------------------------------------------------------------------------
def quantize_vector(params_head, x, bits: int = 3, rot: int = 0):
    """-> (codes uint8[d], norm16 bits, overflow flag, z fp64[d])."""
    ph, x = _f64(params_head), _f64(x)
    d = x.shape[0]
    codes = np.zeros(d, dtype=np.uint8)
    n16 = ctypes.c_uint16(0)
    z = np.zeros(d)
    ov = lib().ref_quantize_vector_v(bits, rot, _ptr(ph), _ptr(x), d, _ptr(codes),
                                     ctypes.byref(n16), _ptr(z))
    return codes, int(n16.value), int(ov), z


def pack_codes(codes, bits: int = 3) -> np.ndarray:
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    d = codes.shape[0]
    out = np.zeros(bits * d // 8, dtype=np.uint8)
    lib().ref_pack_codes_v(bits, _ptr(codes), d, _ptr(out))
    return out


def unpack_codes(packed, d: int, bits: int = 3) -> np.ndarray:
    packed = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    codes = np.zeros(d, dtype=np.uint8)
    lib().ref_unpack_codes_v(bits, _ptr(packed), d, _ptr(codes))
    return codes


def v_put_codes(region, slot: int, codes, bits: int = 3, page: int = 64) -> None:
    """Write one slot's V codes into a page's V region (uint8, modified in place): the 3-bit
    V tile layout, or the slot's record at 2 and 4 bits."""
    assert region.dtype == np.uint8 and region.flags.c_contiguous
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    lib().ref_v_put_codes(bits, codes.shape[0], page, _ptr(region), int(slot), _ptr(codes))


def v_get_codes(region, slot: int, d: int, bits: int = 3, page: int = 64) -> np.ndarray:
    region = np.ascontiguousarray(np.asarray(region, dtype=np.uint8))
    codes = np.zeros(d, np.uint8)
    lib().ref_v_get_codes(bits, d, page, _ptr(region), int(slot), _ptr(codes))
    return codes


def v_region_records(regions, d: int, bits: int = 3, page: int = 64) -> np.ndarray:
    """V regions [..., page * bits*d/8] -> per-slot records [..., page, bits*d/8] in the
    record packing of pack_codes."""
    regions = np.ascontiguousarray(np.asarray(regions, dtype=np.uint8))
    cb = bits * d // 8
    lead = regions.shape[:-1]
    flat = regions.reshape(-1, page * cb)
    out = np.zeros((flat.shape[0], page, cb), np.uint8)
    for i in range(flat.shape[0]):
        lib().ref_v_region_records(bits, d, page, _ptr(flat[i]), _ptr(out[i]))
    return out.reshape(lead + (page, cb))


def block_bytes(d: int, page: int = 64, bits: int = 3) -> int:
    return int(lib().ref_block_bytes_v(bits, d, page))


def quantize_append(params64, d, n_kv_heads, page, blocks, page_table, K, V, seq_ids,
                    positions, bits: int = 3, rot: int = 0) -> int:
    """Quantise K, V ([n_tokens][n_kv_heads][d]) into ``blocks`` (uint8, modified in place).
    Returns the number of saturated norms."""
    assert blocks.dtype == np.uint8 and blocks.flags.c_contiguous
    pt = _i32(page_table)
    K, V = _f64(K), _f64(V)
    sid, pos = _i32(seq_ids), _i32(positions)
    return int(lib().ref_quantize_append_v(bits, rot, _ptr(_f64(params64)), d, n_kv_heads,
                                           page, _ptr(blocks), _ptr(pt), pt.shape[-1], _ptr(K),
                                           _ptr(V), K.shape[0], _ptr(sid), _ptr(pos)))


def dequantize_slot(params64, d, n_kv_heads, page, blocks, phys_page, kv_head, slot,
                    kind, bits: int = 3, rot: int = 0) -> np.ndarray:
    out = np.zeros(d)
    lib().ref_dequantize_slot_v(bits, rot, _ptr(_f64(params64)), d, n_kv_heads, page,
                                _ptr(np.ascontiguousarray(blocks)), phys_page, kv_head, slot,
                                kind, _ptr(out))
    return out


def decode_attention(params64, d, n_kv_heads, page, blocks, page_table, seq_lens, Q, scale,
                     sel=None, bits: int = 3, rot: int = 0) -> np.ndarray:
    """Decode attention on the packed cache.  Q: [n_seqs][n_q_heads][d].  ``sel``: optional
    list of (seq, q_head) pairs to compute (others stay NaN)."""
    Q = _f64(Q)
    n_seqs, n_q_heads = Q.shape[0], Q.shape[1]
    pt = _i32(page_table)
    sl = _i32(seq_lens)
    out = np.full(Q.shape, np.nan)
    selp, nsel = None, 0
    if sel is not None:
        sa = _i32(np.asarray(sel).reshape(-1, 2))
        selp, nsel = _ptr(sa), sa.shape[0]
    lib().ref_decode_attention_v(bits, rot, _ptr(_f64(params64)), d, n_kv_heads, page,
                                 _ptr(np.ascontiguousarray(blocks)), _ptr(pt), pt.shape[-1],
                                 n_seqs, n_q_heads, _ptr(sl), _ptr(Q), float(scale), _ptr(out),
                                 selp, nsel)
    return out


def attention_full(K, V, Q, scale) -> np.ndarray:
    """Full-precision attention for one sequence: K, V [n_tok][n_kv][d], Q [n_q][d]."""
    K, V, Q = _f64(K), _f64(V), _f64(Q)
    n_tok, n_kv, d = K.shape
    out = np.zeros((Q.shape[0], d))
    lib().ref_attention_full(d, n_kv, Q.shape[0], n_tok, _ptr(K), _ptr(V), _ptr(Q),
                             float(scale), _ptr(out))
    return out


def quantize_rows(params64, X, with_dist: bool = True, bits: int = 3, rot: int = 0):
    """Quantise X [n_rows][n_kv_heads][d] (head h with params64[h]).
    -> (codes uint8 [n][H][d], norms uint16 [n][H], dist fp64 [n][H][d] or None), where
    dist is the distance of u to the nearest threshold."""
    X = _f64(X)
    n, H, d = X.shape
    codes = np.zeros((n, H, d), np.uint8)
    norms = np.zeros((n, H), np.uint16)
    dist = np.zeros((n, H, d)) if with_dist else None
    lib().ref_quantize_rows_v(bits, rot, _ptr(_f64(params64)), d, H, _ptr(X), n, _ptr(codes),
                              _ptr(norms), _ptr(dist) if with_dist else None)
    return codes, norms, dist


def unpack_codes_batch(packed, d: int, bits: int = 3) -> np.ndarray:
    """packed uint8 [..., bits*d/8] -> codes uint8 [..., d]."""
    packed = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    lead = packed.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    codes = np.zeros(lead + (d,), np.uint8)
    lib().ref_unpack_codes_batch_v(bits, _ptr(packed), d, n, _ptr(codes))
    return codes
