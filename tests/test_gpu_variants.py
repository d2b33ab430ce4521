"""GPU parity of the format variants against the fp64 oracle: 2- and 4-bit Lloyd-Max
codebooks and the SO(2) (PlanarQuant) rotation, through the same C ABI as the method.
Codes bit-exact outside the 1e-6 band, norms within 1 ulp, decode and multi-token
attention within 2e-3 relative L2 of the oracle run on the GPU's own packed cache."""
import numpy as np
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl
from _gpu_util import ATTN_TOL, Run, check_attention, codes_all, log_record

pytestmark = pytest.mark.gpu

VARIANTS = [(2, 0), (4, 0), (3, 1), (2, 1), (4, 1)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _tokens(cfg):
    seqs, pos = [], []
    for s, n in enumerate(cfg.prefill_lens()):
        seqs.append(np.full(n, s))
        pos.append(np.arange(n))
    return np.concatenate(seqs), np.concatenate(pos)


@pytest.mark.parametrize("bits,rot", VARIANTS)
def test_variant_quantize_and_decode_match_oracle(oracle, bits, rot):
    cfg = wl.small_variant(wl.workload(2), length=1500)       # Student-t, channel scales
    run = Run(cfg, bits=bits, rot=rot)
    assert iq.isoq_params_format(run.params) == (bits, rot)
    run.prefill()
    seqs, pos = _tokens(cfg)
    log_record({"case": f"var_b{bits}_r{rot}_codes", **codes_all(oracle, run, seqs, pos)})
    Q, out = run.decode()
    torch.cuda.synchronize()
    stats = check_attention(oracle, run, Q, out, cfg.decode_lens())
    log_record({"case": f"var_b{bits}_r{rot}_attention", **stats})
    assert iq.isoq_get_status(run.cache) == 0


@pytest.mark.parametrize("bits,rot", [(2, 1), (4, 0)])
def test_variant_batched_paged_and_outliers(oracle, bits, rot):
    """Shuffled pages, ragged lengths and the appended token (workload 4's structure), and
    fp32 inputs with x8 outlier channels (workload 1's)."""
    for cfg in (wl.small_variant(wl.workload(4), n_seqs=3, len_range=(1, 300)),
                wl.workload(1)):
        run = Run(cfg, bits=bits, rot=rot)
        run.prefill()
        run.append()
        seqs, pos = _tokens(cfg)
        codes_all(oracle, run, seqs, pos)
        Q, out = run.decode()
        torch.cuda.synchronize()
        stats = check_attention(oracle, run, Q, out, cfg.decode_lens())
        log_record({"case": f"var_b{bits}_r{rot}_{cfg.name}", **stats})


def test_planar_rotation_at_d256(oracle):
    cfg = wl.small_variant(wl.workload(3), length=600)        # d = 256, RoPE'd K
    run = Run(cfg, bits=3, rot=1)
    run.prefill()
    seqs, pos = _tokens(cfg)
    codes_all(oracle, run, seqs, pos)
    Q, out = run.decode()
    torch.cuda.synchronize()
    log_record({"case": "var_b3_r1_d256", **check_attention(oracle, run, Q, out, cfg.decode_lens())})


def test_variant_multi_token(oracle):
    cfg = wl.small_variant(wl.workload(2), length=700)
    run = Run(cfg, bits=4, rot=1)
    run.prefill()
    n_q = 4
    Q = wl.query_chunk(cfg, n_q, device="cuda")
    L = cfg.decode_lens()[0]
    nb = iq.isoq_multi_token_workspace_bytes(1, n_q, cfg.n_q_heads, cfg.n_kv_heads, cfg.d, L)
    ws = torch.empty((nb,), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, n_q, cfg.n_q_heads, cfg.d), dtype=torch.float32, device="cuda")
    iq.isoq_multi_token_attention(run.params, run.cache, Q, torch.tensor([L], dtype=torch.int32,
                                  device="cuda"), L, out, cfg.scale, ws)
    torch.cuda.synchronize()
    pt = run.layout.page_table.numpy()
    ref = oracle.decode_attention(run.params64(), cfg.d, cfg.n_kv_heads, 64,
                                  run.cache.blocks.cpu().numpy(), np.repeat(pt[:1], n_q, 0),
                                  [L - n_q + i + 1 for i in range(n_q)],
                                  Q[0].float().cpu().numpy().astype(np.float64), cfg.scale,
                                  bits=4, rot=1)
    got = out[0].cpu().numpy().astype(np.float64)
    err = np.linalg.norm(got - ref, axis=-1) / np.linalg.norm(ref, axis=-1)
    assert err.max() <= ATTN_TOL


def test_variant_rejects_unsupported_formats():
    lib = iq.raw_lib()
    h = iq.ctypes.c_void_p()
    assert lib.isoq_make_params_v(0, 256, 2, 2, 0, iq.ctypes.byref(h)) == iq.ISOQ_E_DIM
    with pytest.raises(iq.IsoqError):
        iq.isoq_make_params(0, 128, 2, bits=1)
