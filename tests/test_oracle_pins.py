"""Pins for the fp64 oracle: each checks it against something other than itself (a
library routine, a published table, a closed form, brute force), chosen so that a
plausible slip in the oracle (a dropped term, a sign, an index, a transposed operand,
a wrong component order) fails at least one of them.

Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
Compressed-Space Attention", Abstract (WHT, block-diagonal SO(4), 3-bit scalar
quantisation, attention on the packed cache; 256 parameters per head vs 16,384 dense).
"""
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats
from scipy.spatial.transform import Rotation

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------------------------
# Random parameters: SplitMix64 + Box-Muller
# ------------------------------------------------------------------------------------
def test_splitmix64_published_vectors(oracle):
    for row in _golden("splitmix64_vectors.txt"):
        seed, n = int(row[0]), int(row[1])
        want = [int(v) for v in row[2:2 + n]]
        got = [int(v) for v in oracle.splitmix64_stream(seed, n)]
        assert got == want


def test_box_muller_is_standard_normal(oracle):
    z = oracle.normals(7, 200_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.var() - 1.0) < 0.01
    assert scipy.stats.kstest(z, "norm").pvalue > 1e-3


def test_params_count_and_unit_quaternions(oracle):
    for d, per_head in ((128, 256), (256, 512)):
        p64, p32 = oracle.make_params(0, d, 3)
        assert p64[0].size == per_head          # 256 stored parameters per head at d=128
        assert np.allclose(np.linalg.norm(p64, axis=-1), 1.0, atol=1e-15)
        assert np.array_equal(p32, p64.astype(np.float32))
    assert 128 * 128 == 16384                     # the dense rotation it is compared with


def test_params_haar_moments(oracle):
    p64, _ = oracle.make_params(123, 256, 64)   # 64 heads x 64 blocks x 2 quaternions
    q = p64.reshape(-1, 4)
    assert np.all(np.abs(q.mean(axis=0)) < 0.02)
    # uniform on S^3: each squared component has mean 1/4, pairwise uncorrelated
    assert np.allclose((q ** 2).mean(axis=0), 0.25, atol=0.01)
    c = np.corrcoef(q.T)
    assert np.all(np.abs(c - np.eye(4)) < 0.03)


def test_params_seed_sensitivity(oracle):
    a, _ = oracle.make_params(0, 128, 2)
    b, _ = oracle.make_params(1, 128, 2)
    assert not np.allclose(a, b)
    # heads draw successive parts of one stream
    c, _ = oracle.make_params(0, 128, 1)
    assert np.array_equal(a[0], c[0])


# ------------------------------------------------------------------------------------
# Walsh-Hadamard transform
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("d", [4, 8, 16, 32, 128, 256])
def test_wht_matches_sylvester_hadamard(oracle, d):
    H = scipy.linalg.hadamard(d).astype(np.float64)      # natural (Sylvester) order
    W = oracle.wht(np.eye(d))                             # row j = WHT(e_j)
    assert np.allclose(W.T, H / math.sqrt(d), atol=1e-15)
    Hu = np.rint(W * math.sqrt(d))                        # the unnormalised +-1 matrix
    assert np.array_equal(np.abs(Hu), np.ones((d, d)))
    assert np.array_equal(Hu @ Hu, d * np.eye(d))         # H.H = d.I exactly


@pytest.mark.parametrize("d", [4, 128, 256])
def test_wht_self_inverse_and_e0(oracle, d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal(d)
    assert np.allclose(oracle.wht(oracle.wht(x)), x, atol=1e-14)
    e0 = np.zeros(d)
    e0[0] = 1
    assert np.allclose(oracle.wht(e0), np.full(d, 1 / math.sqrt(d)), atol=1e-16)


# ------------------------------------------------------------------------------------
# Quaternions and SO(4) blocks
# ------------------------------------------------------------------------------------
def _wxyz_to_xyzw(q):
    return np.array([q[1], q[2], q[3], q[0]])


def _xyzw_to_wxyz(q):
    return np.array([q[3], q[0], q[1], q[2]])


def test_quaternion_units(oracle):
    one, i, j, k = np.eye(4)
    assert np.array_equal(oracle.quat_mul(i, j), k)      # ij = k (Hamilton)
    assert np.array_equal(oracle.quat_mul(j, k), i)
    assert np.array_equal(oracle.quat_mul(k, i), j)
    assert np.array_equal(oracle.quat_mul(j, i), -k)
    assert np.array_equal(oracle.quat_mul(i, i), -one)
    assert np.array_equal(oracle.quat_mul(one, k), k)


def test_quaternion_product_is_rotation_composition(oracle):
    """scipy composes rotations R(a)R(b) = R(a*b) (Hamilton); the product quaternion is
    fixed up to sign."""
    rng = np.random.default_rng(1)
    for _ in range(50):
        a = rng.standard_normal(4)
        b = rng.standard_normal(4)
        a /= np.linalg.norm(a)
        b /= np.linalg.norm(b)
        ra = Rotation.from_quat(_wxyz_to_xyzw(a))
        rb = Rotation.from_quat(_wxyz_to_xyzw(b))
        want = _xyzw_to_wxyz((ra * rb).as_quat())
        got = oracle.quat_mul(a, b)
        assert min(np.abs(got - want).max(), np.abs(got + want).max()) < 1e-14


def test_so4_with_p_equal_q_rotates_vector_part(oracle):
    """x -> p x conj(p) fixes the real axis and rotates the vector part as scipy's rotation
    of the same quaternion (closed form: Rodrigues)."""
    rng = np.random.default_rng(2)
    for _ in range(50):
        p = rng.standard_normal(4)
        p /= np.linalg.norm(p)
        v = rng.standard_normal(3)
        z = oracle.so4_forward(p, p, np.concatenate([[0.0], v]))
        want = Rotation.from_quat(_wxyz_to_xyzw(p)).apply(v)
        assert abs(z[0]) < 1e-15
        assert np.allclose(z[1:], want, atol=1e-14)
        assert np.allclose(oracle.so4_forward(p, p, [1.0, 0, 0, 0]), [1.0, 0, 0, 0], atol=1e-15)


def test_so4_identity_and_left_isoclinic(oracle):
    one = np.array([1.0, 0, 0, 0])
    rng = np.random.default_rng(3)
    y = rng.standard_normal(4)
    assert np.allclose(oracle.so4_forward(one, one, y), y, atol=0)
    # q = 1: z = p * y, left multiplication == rotation composition for unit y
    p = rng.standard_normal(4)
    p /= np.linalg.norm(p)
    u = y / np.linalg.norm(y)
    want = _xyzw_to_wxyz((Rotation.from_quat(_wxyz_to_xyzw(p)) *
                          Rotation.from_quat(_wxyz_to_xyzw(u))).as_quat())
    got = oracle.so4_forward(p, one, u)
    assert min(np.abs(got - want).max(), np.abs(got + want).max()) < 1e-14
    # p = 1: z = y * conj(q)
    q = rng.standard_normal(4)
    q /= np.linalg.norm(q)
    want = _xyzw_to_wxyz((Rotation.from_quat(_wxyz_to_xyzw(u)) *
                          Rotation.from_quat(_wxyz_to_xyzw(q)).inv()).as_quat())
    got = oracle.so4_forward(one, q, u)
    assert min(np.abs(got - want).max(), np.abs(got + want).max()) < 1e-14


def test_so4_blocks_orthogonal_det1_invertible(oracle):
    p64, _ = oracle.make_params(0, 128, 2)
    for h in range(2):
        for b in range(32):
            p, q = p64[h, b, 0], p64[h, b, 1]
            M = np.stack([oracle.so4_forward(p, q, e) for e in np.eye(4)], axis=1)
            assert np.abs(M.T @ M - np.eye(4)).max() <= 1e-12
            assert abs(np.linalg.det(M) - 1.0) <= 1e-12
            y = np.random.default_rng(b).standard_normal(4)
            assert np.allclose(oracle.so4_inverse(p, q, oracle.so4_forward(p, q, y)), y,
                               atol=1e-14)


def test_full_rotation_orthogonal_and_preserves_dot(oracle):
    """R = blockdiag(SO(4)) . WHT is orthogonal: (Rq).(Rk) = q.k, and unrotate inverts."""
    d = 128
    p64, _ = oracle.make_params(0, d, 1)
    rng = np.random.default_rng(4)
    for _ in range(20):
        q, k = rng.standard_normal(d), rng.standard_normal(d) * 3
        rq, rk = oracle.rotate(p64[0], q), oracle.rotate(p64[0], k)
        assert abs(rq @ rk - q @ k) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(k)
        assert np.allclose(oracle.unrotate(p64[0], rk), k, atol=1e-13)
    R = np.stack([oracle.rotate(p64[0], e) for e in np.eye(d)], axis=1)
    assert np.abs(R.T @ R - np.eye(d)).max() < 1e-13
    assert abs(np.linalg.det(R) - 1.0) < 1e-10
    # R is WHT followed by blocks: R applied to H's columns is block-diagonal
    B = R @ (scipy.linalg.hadamard(d) / math.sqrt(d))      # = blockdiag(M_b) (WHT^-1 = WHT)
    mask = np.kron(np.eye(d // 4), np.ones((4, 4))).astype(bool)
    assert np.abs(B[~mask]).max() < 1e-14


# ------------------------------------------------------------------------------------
# Codebook
# ------------------------------------------------------------------------------------
def test_codebook_against_max_1960(oracle):
    L, T = oracle.levels(), oracle.thresholds()
    assert np.array_equal(L, -L[::-1])                  # symmetric
    assert np.all(np.diff(L) > 0)                       # ascending codes
    for kind, idx, val in _golden("lloyd_max_gaussian_n8.txt"):
        idx, val = int(idx), float(val)
        if kind == "level":
            assert abs(L[4 + idx] - val) < 5e-4
        elif kind == "threshold":
            assert abs(T[3 + idx] - val) < 5e-4


def test_codebook_lloyd_max_conditions(oracle):
    """Centroid condition: each level is E[u | u in its cell] for u ~ N(0,1); thresholds are
    midpoints; the distortion equals Max's 0.03454."""
    L, T = oracle.levels(), oracle.thresholds()
    edges = np.concatenate([[-np.inf], T, [np.inf]])
    phi, Phi = scipy.stats.norm.pdf, scipy.stats.norm.cdf
    for c in range(8):
        a, b = edges[c], edges[c + 1]
        centroid = (phi(a) - phi(b)) / (Phi(b) - Phi(a))
        assert abs(centroid - L[c]) < 1e-4
    assert np.allclose(T, 0.5 * (L[:-1] + L[1:]), atol=0)
    mse = sum(scipy.integrate.quad(lambda u, c=c: (u - L[c]) ** 2 * phi(u), edges[c],
                                   edges[c + 1])[0] for c in range(8))
    want = float([r for r in _golden("lloyd_max_gaussian_n8.txt") if r[0] == "mse"][0][2])
    assert abs(mse - want) < 5e-5


# ------------------------------------------------------------------------------------
# Quantiser
# ------------------------------------------------------------------------------------
def test_codes_are_nearest_level(oracle):
    """Brute force: the code is the index of the nearest level to u = sqrt(d) z / ||x||."""
    L = oracle.levels()
    p64, _ = oracle.make_params(0, 128, 1)
    rng = np.random.default_rng(5)
    for _ in range(100):
        x = rng.standard_normal(128) * rng.uniform(0.01, 100)
        codes, n16, ov, z = oracle.quantize_vector(p64[0], x)
        u = math.sqrt(128) * z / np.linalg.norm(x)
        nearest = np.argmin(np.abs(u[:, None] - L[None, :]), axis=1)
        assert np.array_equal(codes, nearest)
        assert np.allclose(z, oracle.rotate(p64[0], x), atol=0)


def test_norm_is_fp16_of_l2(oracle):
    p64, _ = oracle.make_params(0, 128, 1)
    rng = np.random.default_rng(6)
    for _ in range(200):
        x = rng.standard_normal(128) * rng.uniform(1e-3, 1e3)
        _, n16, ov, _ = oracle.quantize_vector(p64[0], x)
        assert ov == 0
        assert n16 == int(np.array(np.linalg.norm(x), dtype=np.float16).view(np.uint16))


def test_zero_vector_and_saturation(oracle):
    p64, _ = oracle.make_params(0, 128, 1)
    codes, n16, ov, _ = oracle.quantize_vector(p64[0], np.zeros(128))
    assert n16 == 0 and ov == 0 and np.all(codes == 4)       # level +0.2451 (tie rounds up)
    codes, n16, ov, _ = oracle.quantize_vector(p64[0], np.full(128, 1e4))
    assert n16 == 0x7BFF and ov == 1                          # 65504, flagged
    x = np.zeros(128)
    x[0] = 65519.0                                             # rounds down to 65504: no flag
    _, n16, ov, _ = oracle.quantize_vector(p64[0], x)
    assert n16 == 0x7BFF and ov == 0


def test_fp16_rounding_matches_numpy(oracle):
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.uniform(-9, 5, 2000),
        [0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0],
    ])
    for v in vals:
        with np.errstate(over="ignore"):
            want = int(np.array(v, dtype=np.float16).view(np.uint16))
        assert oracle.fp16_bits(v) == want, v
        h = oracle.fp16_bits(v)
        if (h & 0x7C00) != 0x7C00:
            assert oracle.fp16_value(h) == float(np.array(want, np.uint16).view(np.float16))


def test_isotropy_of_rotated_coordinates(oracle):
    """The rotation spreads outlier channels: with 4 channels x8 the raw per-channel
    variance ratio is ~64, after WHT + SO(4) the per-coordinate variance of u is flat."""
    d, n = 128, 1024
    p64, _ = oracle.make_params(0, d, 1)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((n, d))
    x[:, rng.choice(d, 4, replace=False)] *= 8
    u = np.stack([math.sqrt(d) * oracle.rotate(p64[0], r) / np.linalg.norm(r) for r in x])
    raw = x.var(axis=0)
    rot = u.var(axis=0)
    assert raw.max() / raw.min() > 20
    assert rot.max() / rot.min() < 1.5


def test_quantisation_mse_matches_lloyd_max(oracle):
    """Relative reconstruction error ||x - x_hat||^2 / ||x||^2 on Gaussian vectors is the
    quantiser's distortion per coordinate (~0.0345)."""
    d = 128
    p64, _ = oracle.make_params(0, d, 1)
    L = oracle.levels()
    rng = np.random.default_rng(9)
    errs = []
    for _ in range(400):
        x = rng.standard_normal(d)
        codes, n16, _, _ = oracle.quantize_vector(p64[0], x)
        xh = oracle.unrotate(p64[0], oracle.fp16_value(n16) / math.sqrt(d) * L[codes])
        errs.append(np.sum((x - xh) ** 2) / np.sum(x ** 2))
    assert abs(np.mean(errs) - 0.0345) < 0.003


# ------------------------------------------------------------------------------------
# Packing
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("d", [32, 128, 256])
def test_pack_roundtrip_every_code_every_position(oracle, d):
    rng = np.random.default_rng(d)
    assert oracle.pack_codes(np.zeros(d, np.uint8)).shape == (3 * d // 8,)   # 48 B at d=128
    for i in range(d):
        for c in range(8):
            codes = rng.integers(0, 8, d).astype(np.uint8)
            codes[i] = c
            assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(codes), d), codes)


def test_pack_is_bijective_on_bytes(oracle):
    rng = np.random.default_rng(10)
    for _ in range(200):
        b = rng.integers(0, 256, 48).astype(np.uint8)
        assert np.array_equal(oracle.pack_codes(oracle.unpack_codes(b, 128)), b)


def test_pack_single_code_bit_positions(oracle):
    """Each of the 3d bits of a vector's codes lands on its own bit of the 3d/8 bytes."""
    d = 128
    seen = np.zeros(3 * d, dtype=int)
    for i in range(d):
        for b in range(3):
            codes = np.zeros(d, np.uint8)
            codes[i] = 1 << b
            bits = np.unpackbits(oracle.pack_codes(codes), bitorder="little")
            assert bits.sum() == 1
            seen += bits
    assert np.all(seen == 1)


# ------------------------------------------------------------------------------------
# Decode attention on the packed cache
# ------------------------------------------------------------------------------------
def _tiny_cache(oracle, d, n_kv, G, lens, seed, page=64, shuffle=True, outliers=False):
    rng = np.random.default_rng(seed)
    p64, p32 = oracle.make_params(seed, d, n_kv)
    pp = p32.astype(np.float64)
    npg = [(n + page - 1) // page for n in lens]
    ids = rng.permutation(sum(npg)) if shuffle else np.arange(sum(npg))
    pt = np.full((len(lens), max(npg)), -1, np.int32)
    o = 0
    for s, n in enumerate(npg):
        pt[s, :n] = ids[o:o + n]
        o += n
    blocks = np.zeros(sum(npg) * n_kv * oracle.block_bytes(d, page), np.uint8)
    KV = []
    for s, n in enumerate(lens):
        K = rng.standard_normal((n, n_kv, d))
        V = rng.standard_normal((n, n_kv, d))
        if outliers:
            K[..., :4] *= 8
        oracle.quantize_append(pp, d, n_kv, page, blocks, pt, K, V, np.full(n, s, np.int32),
                               np.arange(n, dtype=np.int32))
        KV.append((K, V))
    Q = rng.standard_normal((len(lens), n_kv * G, d))
    return pp, pt, blocks, KV, Q


def test_decode_rotated_space_equals_materialised(oracle):
    """Attention computed in the rotated space on codes equals softmax attention over the
    explicitly dequantised K-hat = R^T (n/sqrt(d)) L[c] (and V-hat)."""
    d, n_kv, G, page = 128, 2, 4, 64
    lens = [1, 63, 64, 65, 200]
    pp, pt, blocks, _, Q = _tiny_cache(oracle, d, n_kv, G, lens, 11)
    scale = 1 / math.sqrt(d)
    out = oracle.decode_attention(pp, d, n_kv, page, blocks, pt, lens, Q, scale)
    for s, n in enumerate(lens):
        for h in range(n_kv * G):
            kvh = h // G
            Kh = np.stack([oracle.dequantize_slot(pp, d, n_kv, page, blocks, pt[s, t // page],
                                                  kvh, t % page, 0) for t in range(n)])
            Vh = np.stack([oracle.dequantize_slot(pp, d, n_kv, page, blocks, pt[s, t // page],
                                                  kvh, t % page, 1) for t in range(n)])
            sc = scale * Kh @ Q[s, h]
            p = np.exp(sc - sc.max())
            want = (p / p.sum()) @ Vh
            assert np.allclose(out[s, h], want, atol=1e-12 * max(1, np.abs(want).max()))


def test_decode_single_token_returns_its_value(oracle):
    d, n_kv, G, page = 128, 1, 2, 64
    pp, pt, blocks, _, Q = _tiny_cache(oracle, d, n_kv, G, [1], 12)
    out = oracle.decode_attention(pp, d, n_kv, page, blocks, pt, [1], Q, 0.1)
    v = oracle.dequantize_slot(pp, d, n_kv, page, blocks, pt[0, 0], 0, 0, 1)
    assert np.allclose(out[0, 0], v, atol=1e-13) and np.allclose(out[0, 1], v, atol=1e-13)


def test_decode_empty_sequence_is_zero(oracle):
    d, n_kv, G, page = 128, 1, 1, 64
    pp, pt, blocks, _, Q = _tiny_cache(oracle, d, n_kv, G, [64, 5], 13)
    out = oracle.decode_attention(pp, d, n_kv, page, blocks, pt, [0, 5], Q, 0.1)
    assert np.array_equal(out[0, 0], np.zeros(d))
    assert np.all(np.isfinite(out[1, 0]))


def test_decode_gqa_head_mapping(oracle):
    """Query head h reads KV head h // G: duplicating a query across heads of one group
    gives identical outputs, across groups different ones."""
    d, n_kv, G, page = 128, 2, 4, 64
    pp, pt, blocks, _, Q = _tiny_cache(oracle, d, n_kv, G, [130], 14)
    Q[0, :] = Q[0, 0]
    out = oracle.decode_attention(pp, d, n_kv, page, blocks, pt, [130], Q, 0.1)
    assert np.allclose(out[0, 1], out[0, 0], atol=0) and np.allclose(out[0, 3], out[0, 0], atol=0)
    assert not np.allclose(out[0, 4], out[0, 0])


def test_decode_page_table_indirection(oracle):
    """Same data under a shuffled and an identity page table gives the same attention."""
    d, n_kv, G, page = 128, 2, 2, 64
    lens = [150, 64]
    a = _tiny_cache(oracle, d, n_kv, G, lens, 15, shuffle=True)
    b = _tiny_cache(oracle, d, n_kv, G, lens, 15, shuffle=False)
    oa = oracle.decode_attention(a[0], d, n_kv, page, a[2], a[1], lens, a[4], 0.1)
    ob = oracle.decode_attention(b[0], d, n_kv, page, b[2], b[1], lens, b[4], 0.1)
    assert np.array_equal(oa, ob)
    assert not np.array_equal(a[2], b[2])


@pytest.mark.parametrize("d", [4, 8, 16])
def test_tiny_attention_brute_force_error_bound(oracle, d):
    """Tiny d (no packing): dequantised attention vs full precision, brute force.  The
    output error stays within 3 x sqrt(measured quantisation MSE)."""
    rng = np.random.default_rng(d)
    p64, _ = oracle.make_params(d, d, 1)
    L = oracle.levels()
    n = 48
    K, V = rng.standard_normal((n, 1, d)), rng.standard_normal((n, 1, d))
    q = rng.standard_normal((1, d))

    def deq(x):
        codes, n16, _, _ = oracle.quantize_vector(p64[0], x)
        return oracle.unrotate(p64[0], oracle.fp16_value(n16) / math.sqrt(d) * L[codes])

    Kh = np.stack([deq(k[0]) for k in K])[:, None, :]
    Vh = np.stack([deq(v[0]) for v in V])[:, None, :]
    mse = np.mean(np.sum((Kh - K) ** 2, -1) / np.sum(K ** 2, -1))
    full = oracle.attention_full(K, V, q, 1 / math.sqrt(d))
    quant = oracle.attention_full(Kh, Vh, q, 1 / math.sqrt(d))
    # brute force: explicit softmax
    sc = (K[:, 0] @ q[0]) / math.sqrt(d)
    p = np.exp(sc - sc.max())
    assert np.allclose(full[0], (p / p.sum()) @ V[:, 0], atol=1e-13)
    rel = np.linalg.norm(quant - full) / np.linalg.norm(full)
    assert rel <= 3 * math.sqrt(mse)


def test_attention_vs_full_precision_config1_like(oracle):
    """d=128 through the packed cache, 4 outlier channels x8: output error relative to full
    precision is bounded by 3 sqrt(MSE) (near-zero degradation claim, as a ratio)."""
    d, n_kv, G, page = 128, 2, 4, 64
    pp, pt, blocks, KV, Q = _tiny_cache(oracle, d, n_kv, G, [512], 16, outliers=True)
    scale = 1 / math.sqrt(d)
    out = oracle.decode_attention(pp, d, n_kv, page, blocks, pt, [512], Q, scale)
    K, V = KV[0]
    full = oracle.attention_full(K, V, Q[0], scale)
    rel = np.linalg.norm(out[0] - full) / np.linalg.norm(full)
    assert rel < 3 * math.sqrt(0.0345)
