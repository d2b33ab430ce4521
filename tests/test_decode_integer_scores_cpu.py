"""The 3-bit decode's integer score arithmetic, restated on the CPU in int64.

The decode kernel scores a token as sum_i q_i L[c_i] on s8 tensor-core products: each level
is an integer 10000 L[c] = kh * 256 + kl split into two signed bytes, the rotated query row is
scaled to a 24-bit integer and split into three balanced signed digits (d2, d1, d0), and the
two s32 accumulators C1 = [d2.kh ; d1.kh] and C2 = [d2.kl ; d1.kl + d0.kh] are combined as
raw = (256 C1_top + C2_top + C1_bot) + C2_bot / 256, which is the integer score / 2^16 minus
only the d0.kl term.  These tests read the constants from the kernel source and check what the
scheme needs to be exact: every digit and level byte fits s8, no s32 accumulator can
overflow at d = 128 or 256, the combination drops exactly d0.kl / 2^16, and the score's
relative error is far inside the 2e-3 attention tolerance.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "rotated_bit_kv_isoquant_b200", "csrc", "isoq_decode_i8.cu")

# Lloyd-Max levels of N(0,1) for 8 levels, ascending (the codebook the format states)
LEVELS = np.array([-2.1520, -1.3440, -0.7560, -0.2451, 0.2451, 0.7560, 1.3440, 2.1520])


def _source_constants():
    src = open(SRC).read()
    qmax = float(re.search(r"kQMax\s*=\s*([0-9.eE+]+)f", src).group(1))
    lscale = float(re.search(r"kLevelScale\s*=\s*([0-9.eE+]+)f", src).group(1))
    body = re.search(r"constexpr int ilevel\(int c\) \{(.*?)\}", src, re.S).group(1)
    # "c == 0 ? v0 : c == 1 ? v1 : ... : v7;"
    ints = [int(x) for x in re.findall(r"\?\s*(-?\d+)", body)]
    ints += [int(x) for x in re.findall(r":\s*(-?\d+)\s*;", body)]
    return qmax, lscale, np.array(ints, dtype=np.int64)


def _split_level(v):
    """kh = floor((v + 128) / 256), kl = v - 256 kh (kl in [-128, 127])."""
    kh = np.floor_divide(v + 128, 256)
    return kh, v - 256 * kh


def _digits3(q):
    """Balanced base-256 digits: q = d2 65536 + d1 256 + d0, each in [-128, 127]."""
    d0 = ((q + 128) & 255) - 128
    r = (q - d0) >> 8
    d1 = ((r + 128) & 255) - 128
    d2 = (r - d1) >> 8
    return d2, d1, d0


def test_integer_levels_match_the_codebook():
    qmax, lscale, il = _source_constants()
    assert lscale == 1.0e4 and len(il) == 8
    assert np.array_equal(il, np.round(LEVELS * lscale).astype(np.int64))
    kh, kl = _split_level(il)
    assert np.all((kl >= -128) & (kl <= 127)) and np.all((kh >= -128) & (kh <= 127))
    assert np.array_equal(kh * 256 + kl, il)


def test_query_digits_fit_s8_and_recompose():
    qmax, _, _ = _source_constants()
    lim = int(qmax)
    rng = np.random.default_rng(5)
    q = np.concatenate([np.arange(-lim, -lim + 70000), np.arange(lim - 70000, lim + 1),
                        np.arange(-70000, 70000), rng.integers(-lim, lim + 1, 2_000_000)])
    d2, d1, d0 = _digits3(q.astype(np.int64))
    for d in (d2, d1, d0):
        assert d.min() >= -128 and d.max() <= 127
    assert np.array_equal(d2 * 65536 + d1 * 256 + d0, q)


def test_accumulators_cannot_overflow():
    qmax, _, il = _source_constants()
    kh, kl = _split_level(il)
    d2max = int(qmax) // 65536 + 1           # |d2| <= 123 for |q| <= 8e6
    for D in (128, 256):
        c1 = D * d2max * np.abs(kh).max()      # C1 rows: sum over the D dims
        c2 = D * (128 * np.abs(kl).max() + 128 * np.abs(kh).max())
        z = 256 * c1 + c2 + c1                 # the combination before the int->float step
        assert z < 2 ** 31, (D, z)


def test_combination_drops_only_the_lowest_product():
    qmax, _, il = _source_constants()
    kh_t, kl_t = _split_level(il)
    rng = np.random.default_rng(11)
    for D in (128, 256):
        for trial in range(200):
            z = rng.standard_normal(D) * (rng.random() * 10 + 0.1)
            z[rng.integers(0, D)] *= 40.0       # an outlier dim sets the scale
            S = qmax / np.abs(z).max()
            q = np.rint(z * S).astype(np.int64)  # round half to even, as the kernel's rn
            c = rng.integers(0, 8, D)
            d2, d1, d0 = _digits3(q)
            kh, kl = kh_t[c], kl_t[c]
            c1_top, c1_bot = np.dot(d2, kh), np.dot(d1, kh)
            c2_top, c2_bot = np.dot(d2, kl), np.dot(d1, kl) + np.dot(d0, kh)
            raw_times_256 = 256 * (256 * c1_top + c2_top + c1_bot) + c2_bot
            exact = np.dot(q, il[c])               # the full integer score
            assert raw_times_256 * 256 == exact - np.dot(d0, kl)
            # relative to the score scale |q| |L| sqrt(D): the dropped term and the query's
            # rounding to 24 bits are both ~1e-7, four orders inside the 2e-3 tolerance
            ref = np.dot(z, LEVELS[c]) * S * 1e4
            scale = np.linalg.norm(q) * np.linalg.norm(il[c])
            assert abs(raw_times_256 * 256 - ref) <= 1e-6 * scale
