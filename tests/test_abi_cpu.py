"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every entry
point include/isoq.h declares, validates arguments before touching the device, and its
host parameter generator agrees bit for bit with the oracle's independent one."""
import ctypes
import os
import re

import numpy as np
import pytest

import rotated_bit_kv_isoquant_b200 as iq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(isoq_\w+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol():
    names = _declared_functions()
    assert "isoq_decode_attention" in names and "isoq_quantize_append" in names
    lib = ctypes.CDLL(iq.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_checked_build_exports_every_declared_symbol():
    """The bounds-checked variant (build.py --checked) has the same entry points."""
    path = os.path.join(ROOT, "rotated_bit_kv_isoquant_b200", "libisoq_checked.so")
    if not os.path.exists(path):
        pytest.skip("libisoq_checked.so not built")
    lib = ctypes.CDLL(path)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


@pytest.mark.parametrize("seed,d,h", [(0, 128, 2), (0, 128, 8), (0, 256, 8), (12345, 128, 3),
                                      (2**63 + 7, 256, 1)])
def test_params_generator_matches_oracle_bitwise(oracle, seed, d, h):
    lib_params = iq.isoq_params_generate(seed, d, h)
    _, ref32 = oracle.make_params(seed, d, h)
    assert lib_params.shape == ref32.shape
    assert np.array_equal(lib_params.view(np.uint32), ref32.view(np.uint32))
    assert lib_params[0].size == d * 2            # 256 parameters per head at d = 128


def test_params_generate_rejects():
    lib = iq.raw_lib()
    buf = np.zeros(1024, np.float32)
    assert lib.isoq_params_generate(0, 96, 1, buf.ctypes.data) == iq.ISOQ_E_DIM
    assert lib.isoq_params_generate(0, 128, 0, buf.ctypes.data) == iq.ISOQ_E_ARG
    assert lib.isoq_params_generate(0, 128, 1, None) == iq.ISOQ_E_ARG


@pytest.mark.parametrize("seed,d,h", [(0, 128, 8), (99, 256, 3)])
def test_so2_params_generator_matches_oracle_bitwise(oracle, seed, d, h):
    lib_params = iq.isoq_params_generate(seed, d, h, rotation=iq.ISOQ_ROT_SO2)
    _, ref32 = oracle.make_params_so2(seed, d, h)
    assert lib_params.shape == ref32.shape == (h, d // 2, 2)
    assert np.array_equal(lib_params.view(np.uint32), ref32.view(np.uint32))


def test_variant_formats_host_checks():
    assert iq.isoq_block_bytes(128, bits=2) == 2 * 64 * (32 + 2)
    assert iq.isoq_block_bytes(128, bits=4) == 2 * 64 * (64 + 2)
    assert iq.isoq_block_bytes(128, bits=4) % 16 == 0 and iq.isoq_block_bytes(128, bits=2) % 16 == 0
    assert iq.isoq_block_bytes(256, bits=2) == 0          # variants are d = 128 only
    assert iq.isoq_block_bytes(128, bits=5) == 0
    lib = iq.raw_lib()
    h = ctypes.c_void_p()
    # validated before any device call
    assert lib.isoq_make_params_v(0, 128, 2, 5, iq.ISOQ_ROT_SO4, ctypes.byref(h)) == iq.ISOQ_E_DIM
    assert lib.isoq_make_params_v(0, 256, 2, 4, iq.ISOQ_ROT_SO4, ctypes.byref(h)) == iq.ISOQ_E_DIM
    assert lib.isoq_make_params_v(0, 128, 2, 3, 7, ctypes.byref(h)) == iq.ISOQ_E_ARG
    assert lib.isoq_params_format(None, None, None) == iq.ISOQ_E_ARG


def test_block_bytes():
    assert iq.isoq_block_bytes(128) == 6400
    assert iq.isoq_block_bytes(256) == 12544
    assert iq.isoq_block_bytes(128) % 16 == 0 and iq.isoq_block_bytes(256) % 16 == 0
    assert iq.isoq_block_bytes(64) == 0
    assert iq.isoq_block_bytes(128, 32) == 0


def test_split_plan_host_arithmetic():
    # splits cover the context with whole pages; more units -> fewer splits
    for (ns, hq, hkv, d, L) in [(1, 32, 4, 128, 32768), (8, 64, 8, 128, 131072),
                                (64, 32, 8, 128, 65537), (1, 8, 2, 128, 1024), (1, 8, 2, 128, 1),
                                (3, 4, 4, 256, 0)]:
        n = iq.isoq_decode_num_splits(ns, hq, hkv, d, L)
        pages = max(1, -(-L // 64))
        assert 1 <= n <= pages
        ws = iq.isoq_decode_workspace_bytes(ns, hq, hkv, d, L)
        assert ws == ns * hq * n * (d + 4) * 4
    assert iq.raw_lib().isoq_decode_num_splits(1, 6, 4, 128, 100) == iq.ISOQ_E_GQA
    assert iq.raw_lib().isoq_decode_num_splits(1, 8, 4, 96, 100) == iq.ISOQ_E_DIM


def test_split_plan_bounds_chunk_length():
    # a decode chunk is at most 64 pages whatever the batch (a ragged batch is sized by its
    # longest sequence), and at least 16 pages where the context has them
    for (ns, hq, hkv, d, L) in [(64, 32, 8, 128, 65536), (2, 32, 8, 128, 1 << 20),
                                (8, 64, 8, 128, 131072), (1, 32, 4, 128, 32768),
                                (1, 16, 8, 256, 32768)]:
        n = iq.isoq_decode_num_splits(ns, hq, hkv, d, L)
        pages = -(-L // 64)
        pps = -(-pages // n)
        assert pps <= 64, (ns, L, n, pps)
        assert pps >= min(16, pages) or n == 1, (ns, L, n, pps)


def test_argument_validation_without_device():
    lib = iq.raw_lib()
    c = iq.isoq_cache(128, 2, 64, 4, 2, 1, None, None, None)
    # null params / cache pointers are rejected before any CUDA call
    assert lib.isoq_quantize_append(None, ctypes.byref(c), None, None, 0, 1, None, None,
                                    None) == iq.ISOQ_E_ARG
    assert lib.isoq_decode_attention(None, ctypes.byref(c), None, 0, 1, 8, None, 64, None, 1.0,
                                     None, 0, None) == iq.ISOQ_E_ARG
    assert lib.isoq_get_status(None, None) == iq.ISOQ_E_ARG
    assert iq.isoq_error_string(iq.ISOQ_E_WORKSPACE).startswith("workspace")
