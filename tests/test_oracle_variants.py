"""Pins of the oracle's format variants against sources other than the oracle itself:
the 2- and 4-bit Lloyd-Max codebooks (Max 1960 tables, and the Lloyd-Max fixed point
computed here with scipy), brute-force nearest-level quantisation, SO(2) blocks against
complex multiplication, the packed layouts bit by bit, and decode on codes against
softmax attention over explicitly dequantised K-hat / V-hat.

Variants of "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
Compressed-Space Attention", Abstract: the same pipeline with 2 or 4 bits per code (the
"3-4 bit" family), and PlanarQuant read as WHT followed by 2x2 (SO(2)) rotation blocks.
"""
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.stats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
VARIANTS = [(2, 0), (4, 0), (3, 1), (2, 1), (4, 1)]


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _lloyd_max(n_levels, iters=20000):
    """The Lloyd-Max fixed point for N(0,1): levels = conditional means of their cells,
    thresholds = midpoints (Lloyd's method I), iterated from a uniform start."""
    phi, Phi = scipy.stats.norm.pdf, scipy.stats.norm.cdf
    L = np.linspace(-2.0, 2.0, n_levels)
    for _ in range(iters):
        e = np.concatenate([[-np.inf], 0.5 * (L[:-1] + L[1:]), [np.inf]])
        L = (phi(e[:-1]) - phi(e[1:])) / (Phi(e[1:]) - Phi(e[:-1]))
    return L


@pytest.mark.parametrize("bits,name", [(2, "lloyd_max_gaussian_n4.txt"),
                                       (4, "lloyd_max_gaussian_n16.txt")])
def test_codebooks_against_max_1960(oracle, bits, name):
    L, T = oracle.levels(bits), oracle.thresholds(bits)
    n = 1 << bits
    assert L.shape == (n,) and T.shape == (n - 1,)
    assert np.array_equal(L, -L[::-1]) and np.all(np.diff(L) > 0)
    assert np.allclose(T, 0.5 * (L[:-1] + L[1:]), atol=0)
    for kind, idx, val in _golden(name):
        idx, val = int(idx), float(val)
        if kind == "level":
            assert abs(L[n // 2 + idx] - val) < 5e-4
        elif kind == "threshold":
            assert abs(T[n // 2 - 1 + idx] - val) < 5e-4


@pytest.mark.parametrize("bits", [2, 4])
def test_codebooks_are_the_lloyd_max_fixed_point(oracle, bits):
    opt = _lloyd_max(1 << bits)
    assert np.abs(oracle.levels(bits) - opt).max() < 1e-4   # 4-decimal values


def test_two_bit_distortion_matches_max(oracle):
    L, T = oracle.levels(2), oracle.thresholds(2)
    phi = scipy.stats.norm.pdf
    e = np.concatenate([[-np.inf], T, [np.inf]])
    mse = sum(scipy.integrate.quad(lambda u, c=c: (u - L[c]) ** 2 * phi(u), e[c], e[c + 1])[0]
              for c in range(4))
    want = float([r for r in _golden("lloyd_max_gaussian_n4.txt") if r[0] == "mse"][0][2])
    assert abs(mse - want) < 5e-5


# ------------------------------------------------------------------------------------
# SO(2) blocks (PlanarQuant variant)
# ------------------------------------------------------------------------------------
def test_so2_params_are_unit_and_uniform(oracle):
    p64, p32 = oracle.make_params_so2(0, 128, 8)
    assert p64.shape == (8, 64, 2)                   # d/2 angles per head (cos, sin)
    assert np.allclose(p64[..., 0] ** 2 + p64[..., 1] ** 2, 1.0, atol=1e-15)
    assert np.array_equal(p32, p64.astype(np.float32))
    phi = np.mod(np.arctan2(p64[..., 1], p64[..., 0]), 2 * np.pi).ravel() / (2 * np.pi)
    assert scipy.stats.kstest(phi, "uniform").pvalue > 1e-3
    # the stream is SplitMix64: the first angle is 2 pi * (top 53 bits of draw 1) / 2^53
    k = int(oracle.splitmix64_stream(0, 1)[0]) >> 11
    assert math.isclose(p64[0, 0, 0], math.cos(2 * math.pi * k / 2.0 ** 53), abs_tol=1e-15)


def test_so2_block_is_complex_multiplication(oracle):
    rng = np.random.default_rng(3)
    for _ in range(50):
        a = rng.uniform(0, 2 * np.pi)
        cs = np.array([np.cos(a), np.sin(a)])
        y = rng.standard_normal(2)
        w = np.exp(1j * a) * (y[0] + 1j * y[1])
        z = oracle.so2_forward(cs, y)
        assert np.allclose(z, [w.real, w.imag], atol=1e-14)
        assert np.allclose(oracle.so2_inverse(cs, z), y, atol=1e-14)


def test_so2_rotation_is_orthogonal_and_inverted(oracle):
    d = 64
    p64, _ = oracle.make_params_so2(7, d, 1)
    R = np.stack([oracle.rotate(p64[0], e, rot=1) for e in np.eye(d)], axis=1)
    assert np.abs(R.T @ R - np.eye(d)).max() < 1e-12
    assert abs(np.linalg.det(R) - 1.0) < 1e-10
    # removing the WHT leaves 2x2 blocks on the diagonal
    H = oracle.wht(np.eye(d))
    B = R @ H.T
    mask = np.kron(np.eye(d // 2), np.ones((2, 2)))
    assert np.abs(B * (1 - mask)).max() < 1e-12
    x = np.random.default_rng(1).standard_normal(d)
    assert np.allclose(oracle.unrotate(p64[0], oracle.rotate(p64[0], x, rot=1), rot=1), x,
                       atol=1e-13)


# ------------------------------------------------------------------------------------
# Quantiser and packing
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("bits,rot", VARIANTS)
def test_variant_codes_are_nearest_level(oracle, bits, rot):
    d = 128
    L = oracle.levels(bits)
    p64, _ = oracle.make_params_v(0, d, 1, rot)
    rng = np.random.default_rng(11 + bits + 7 * rot)
    for _ in range(40):
        x = rng.standard_normal(d) * rng.uniform(0.1, 10)
        codes, _, _, z = oracle.quantize_vector(p64[0], x, bits=bits, rot=rot)
        u = math.sqrt(d) * z / np.linalg.norm(x)
        assert np.array_equal(codes, np.argmin(np.abs(u[:, None] - L[None, :]), axis=1))
    codes, n16, _, _ = oracle.quantize_vector(p64[0], np.zeros(d), bits=bits, rot=rot)
    assert n16 == 0 and np.all(codes == (1 << (bits - 1)))   # zero vector: first level > 0


@pytest.mark.parametrize("bits", [2, 4])
def test_variant_pack_round_trip_and_bijection(oracle, bits):
    d = 128
    rng = np.random.default_rng(bits)
    for _ in range(20):
        c = rng.integers(0, 1 << bits, d).astype(np.uint8)
        p = oracle.pack_codes(c, bits=bits)
        assert p.shape == (bits * d // 8,)
        assert np.array_equal(oracle.unpack_codes(p, d, bits=bits), c)
        raw = rng.integers(0, 256, bits * d // 8).astype(np.uint8)
        assert np.array_equal(oracle.pack_codes(oracle.unpack_codes(raw, d, bits=bits), bits=bits), raw)


def _word(p, j):
    return int.from_bytes(bytes(p[4 * j:4 * j + 4]), "little")


def test_four_bit_layout_is_sign_magnitude_nibbles(oracle):
    d = 32
    for dim in (0, 5, 8, 31):
        for c, nib in ((15, 7), (8, 0), (7, 8), (0, 15), (10, 2), (5, 10)):
            codes = np.full(d, 8, np.uint8)          # nibble 0 everywhere else
            codes[dim] = c
            p = oracle.pack_codes(codes, bits=4)
            j, k = dim // 8, dim % 8
            words = [_word(p, i) for i in range(d // 8)]
            assert words[j] == nib << (4 * k)
            assert all(w == 0 for i, w in enumerate(words) if i != j)


def test_two_bit_layout_slot_order(oracle):
    d = 32
    slot_of = {}
    for s in range(16):
        dim = 2 * s if s < 4 else (2 * (s - 4) + 1 if s < 8 else (8 + 2 * (s - 8) if s < 12 else 9 + 2 * (s - 12)))
        slot_of[dim] = s
    assert sorted(slot_of) == list(range(16))
    for dim in range(d):
        codes = np.zeros(d, np.uint8)
        codes[dim] = 3
        p = oracle.pack_codes(codes, bits=2)
        j = dim // 16
        assert _word(p, j) == 3 << (2 * slot_of[dim % 16])
        assert _word(p, 1 - j) == 0


# ------------------------------------------------------------------------------------
# Decode on codes equals attention over the materialised K-hat / V-hat
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("bits,rot", VARIANTS)
def test_variant_decode_equals_materialised_attention(oracle, bits, rot):
    d, H, G, n_tok, page = 64, 2, 2, 150, 64
    rng = np.random.default_rng(100 + bits + 10 * rot)
    p64, _ = oracle.make_params_v(5, d, H, rot)
    n_pages = -(-n_tok // page)
    blocks = np.zeros((n_pages, H, oracle.block_bytes(d, page, bits=bits)), np.uint8)
    pt = np.arange(n_pages, dtype=np.int32)[::-1].copy()[None, :]      # reversed pages
    K = rng.standard_normal((n_tok, H, d)) * 2.0
    V = rng.standard_normal((n_tok, H, d))
    oracle.quantize_append(p64, d, H, page, blocks, pt, K, V, np.zeros(n_tok, np.int32),
                           np.arange(n_tok, dtype=np.int32), bits=bits, rot=rot)
    Q = rng.standard_normal((1, H * G, d))
    scale = 1 / math.sqrt(d)
    got = oracle.decode_attention(p64, d, H, page, blocks, pt, [n_tok], Q, scale, bits=bits,
                                  rot=rot)
    Kh = np.zeros((n_tok, H, d))
    Vh = np.zeros((n_tok, H, d))
    for t in range(n_tok):
        for h in range(H):
            ph = int(pt[0, t // page])
            Kh[t, h] = oracle.dequantize_slot(p64, d, H, page, blocks, ph, h, t % page, 0,
                                              bits=bits, rot=rot)
            Vh[t, h] = oracle.dequantize_slot(p64, d, H, page, blocks, ph, h, t % page, 1,
                                              bits=bits, rot=rot)
    want = oracle.attention_full(Kh, Vh, Q[0], scale)
    assert np.abs(got[0] - want).max() < 1e-12


@pytest.mark.parametrize("bits,want", [(2, 0.1175), (4, 0.0095)])
def test_variant_mse_matches_codebook_distortion(oracle, bits, want):
    d = 128
    p64, _ = oracle.make_params(0, d, 1)
    L = oracle.levels(bits)
    rng = np.random.default_rng(13)
    errs = []
    for _ in range(300):
        x = rng.standard_normal(d)
        codes, n16, _, _ = oracle.quantize_vector(p64[0], x, bits=bits)
        xh = oracle.unrotate(p64[0], oracle.fp16_value(n16) / math.sqrt(d) * L[codes])
        errs.append(np.sum((x - xh) ** 2) / np.sum(x ** 2))
    assert abs(np.mean(errs) - want) < 0.08 * want


# ------------------------------------------------------------------------------------
# RoPE of the fused quantize epilogue
# ------------------------------------------------------------------------------------
def test_rope_is_complex_multiplication_by_position_phases(oracle):
    d, base = 128, 10000.0
    rng = np.random.default_rng(21)
    x = rng.standard_normal(d)
    for pos in (0, 1, 7, 1000, 131071):
        got = oracle.rope(x, pos, base)
        theta = base ** (-np.arange(d // 2) * 2.0 / d)
        w = (x[:d // 2] + 1j * x[d // 2:]) * np.exp(1j * pos * theta)
        assert np.allclose(got[:d // 2], w.real, atol=1e-12)
        assert np.allclose(got[d // 2:], w.imag, atol=1e-12)
    assert np.array_equal(oracle.rope(x, 0, base), x)


def test_rope_preserves_norm_and_depends_on_relative_position(oracle):
    d = 64
    rng = np.random.default_rng(22)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    assert abs(np.linalg.norm(oracle.rope(q, 12345)) - np.linalg.norm(q)) < 1e-12
    for m, n in ((10, 3), (500, 499), (70000, 12)):
        lhs = oracle.rope(q, m) @ oracle.rope(k, n)
        rhs = oracle.rope(q, m - n) @ k
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs))
