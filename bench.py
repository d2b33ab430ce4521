"""Benchmark of the IsoQuant packed-KV path on B200: quantize-append + decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 5] [--impl ours|reference]

One step = the whole hot path over one batch of the workload: quantize-append of the full
prefill (in the workload's chunked calls) followed by one decode step of every sequence
on the packed cache.  Default workload: 8 sequences x 131072 tokens, 64 query / 8 KV
heads, d = 128, bf16 K/V quantised in 16384-token chunks (the long-context configuration,
on which both halves of the metric -- quantize Mvec/s and packed-KV decode GB/s -- are
quoted).  Inputs are resident in HBM before the timed region and larger than L2; L2 is
also flushed before each decode.  Timing: CUDA events on the launching stream, barrier +
synchronize around the K timed steps, max over ranks.  Multi-GPU: every rank runs its own
replica (the (sequence, KV head) units are independent), no collective on the data path.

--impl reference times the fp64 CPU oracle (the only reference there is) on a bounded
sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0    # B200 HBM3e specification (context for the measured copy peak)
# the headline metric, printed identically by both arms
METRIC = "packed-KV decode attention GB/s (% of B200 HBM peak); quantize Mvec/s"
# what the decode's contraction computes in (operands and accumulator)
DECODE_DTYPE = "s8xs8->s32 scores (integer codes, 3-digit query), f16xf16->f32 value sum"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the end-to-end timing (default: --steps)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload measurements of the other configurations")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the multi-token and context-parallel measurements")
    ap.add_argument("--chunk", type=int, default=16,
                    help="query tokens per sequence of the multi-token measurement")
    ap.add_argument("--seqs", type=int, default=0,
                    help="use only this many sequences of the workload (small profiling case)")
    return ap.parse_args()


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the slowest rank's time).  One all-reduce
    of a single float after timing; nothing on the data path."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_step_per_rank: float, steps: int, world: int,
                      max_ms: float) -> float:
    """Whole-job rate: every rank processes the same work per step (weak scaling), so the
    job's throughput is all ranks' units divided by the slowest rank's time."""
    return units_per_step_per_rank * steps * world / (max_ms / 1e3)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        if j.get("hbm_gbs"):
            return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _tensor_peak():
    """Dense f16/bf16 tensor peak (TFLOP/s) for a kernel timed alone: the measured burst
    figure, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        if j.get("bf16_tflops"):
            return float(j["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


_KERNEL_SOURCES = {
    # the 3-bit split kernel the decode profiles capture (the combine is < 3% of the call)
    "decode": ["isoq_decode_i8.cu", "isoq_vtile.cuh", "isoq_ptx.cuh", "isoq_common.cuh",
               "isoq_check.cuh", "isoq_internal.h"],
    "quantize": ["isoq_quantize_tc.cu", "isoq_quantize.cu", "isoq_codes.cuh", "isoq_tc.cuh",
                 "isoq_vtile.cuh", "isoq_common.cuh"],
}


def _kernel_sources_sha(kernel: str) -> str:
    """Hash of the sources that build one kernel group (a profile summary records it)."""
    h = hashlib.sha256()
    for name in _KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "rotated_bit_kv_isoquant_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/, if the kernel's
    sources have not changed since (else None)."""
    sha = _kernel_sources_sha(kernel)
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        txt = open(p).read()
        m_k = re.search(r"^kernel_group:\s*(\S+)", txt, re.M)
        m_w = re.search(r"^workload:\s*(\S+)", txt, re.M)
        m_s = re.search(r"^source_sha:\s*(\S+)", txt, re.M)
        m_t = re.search(r"^dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt, re.M)
        if m_k and m_w and m_s and m_t and m_k.group(1) == kernel and m_w.group(1) == workload:
            if m_s.group(1) == sha:
                return float(m_t.group(1))
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            self.out = ""
            return
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.strip()]
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = sorted(sm)[len(sm) // 4:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------------------
# Oracle timing (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------
def oracle_sample(cfg, tokens: int = 4096, units: int = 1):
    """Bounded sample of the workload for the fp64 oracle: the first `tokens` tokens of
    sequence 0 for `units` KV heads (all their query heads), quantised by the oracle into
    its own paged cache, then decoded.  Returns timings and the bytes/vectors processed."""
    import numpy as np
    import torch
    import oracle
    import workloads as wl

    oracle.build()
    K, V = wl.kv_tokens(cfg, 0, 0, tokens, device="cpu")
    H = units
    K = K[:, :H].float().numpy().astype(np.float64)
    V = V[:, :H].float().numpy().astype(np.float64)
    Q = wl.queries(cfg, device="cpu")[:1, :H * cfg.group].float().numpy().astype(np.float64)
    _, p32 = oracle.make_params(wl.PARAM_SEED, cfg.d, H)
    p64 = p32.astype(np.float64)
    npg = -(-tokens // 64)
    pt = np.arange(npg, dtype=np.int32)[None, :]
    blocks = np.zeros(npg * H * oracle.block_bytes(cfg.d), np.uint8)
    t0 = time.perf_counter()
    oracle.quantize_append(p64, cfg.d, H, 64, blocks, pt, K, V, np.zeros(tokens, np.int32),
                           np.arange(tokens, dtype=np.int32))
    t1 = time.perf_counter()
    oracle.decode_attention(p64, cfg.d, H, 64, blocks, pt, [tokens], Q, cfg.scale)
    t2 = time.perf_counter()
    packed = tokens * H * 2 * (3 * cfg.d // 8 + 2)
    return {"quant_s": t1 - t0, "decode_s": t2 - t1, "vectors": tokens * H * 2,
            "packed_bytes": packed, "threads": oracle.num_threads(),
            "pairs": H * cfg.group, "tokens": tokens, "units": H}


def cpu_baseline(cfg, budget_s: float = 12.0, single_core_s: float = 3.0):
    """Oracle decode GB/s (and quantize Mvec/s) on a bounded sample sized to ~budget_s on all
    of the host's cores, and on one core with a sample sized to ~single_core_s."""
    import oracle
    probe = oracle_sample(cfg, tokens=1024, units=1)
    per_tok = (probe["quant_s"] + probe["decode_s"]) / 1024
    tokens = int(max(1024, min(cfg.decode_lens()[0], budget_s / max(per_tok, 1e-9))))
    tokens = (tokens // 64) * 64
    r = oracle_sample(cfg, tokens=tokens, units=1)
    res = {
        "value": r["packed_bytes"] / r["decode_s"] / 1e9, "unit": "GB/s",
        "cores": min(r["threads"], r["pairs"]), "kind": "oracle",
        "quantize_mvec_s": r["vectors"] / r["quant_s"] / 1e6,
        "quantize_cores": r["threads"],
        "sample": (f"sequence 0, first {r['tokens']} tokens, 1 KV head x {r['pairs']} query "
                   f"heads: oracle quantize ({r['vectors']} vectors) then decode "
                   f"({r['packed_bytes']} packed bytes)"),
    }
    if single_core_s > 0:
        threads = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            p1 = oracle_sample(cfg, tokens=256, units=1)
            per1 = (p1["quant_s"] + p1["decode_s"]) / 256
            t1 = int(max(256, min(cfg.decode_lens()[0], single_core_s / max(per1, 1e-9))))
            r1 = oracle_sample(cfg, tokens=(t1 // 64) * 64 or 64, units=1)
        finally:
            oracle.set_num_threads(threads)
        res["single_core"] = {
            "value": r1["packed_bytes"] / r1["decode_s"] / 1e9, "unit": "GB/s", "cores": 1,
            "quantize_mvec_s": r1["vectors"] / r1["quant_s"] / 1e6,
            "sample": f"sequence 0, first {r1['tokens']} tokens, 1 KV head"}
    return res


def run_reference(args, cfg):
    rank, world, _ = _dist_env()
    if rank != 0:
        return 0
    tokens = 2048
    for _ in range(args.warmup):
        oracle_sample(cfg, tokens=tokens)
    dec, qt, rr = 0.0, 0.0, None
    for _ in range(args.steps):
        rr = oracle_sample(cfg, tokens=tokens)
        dec += rr["decode_s"]
        qt += rr["quant_s"]
    value = rr["packed_bytes"] * args.steps / dec / 1e9
    sample = (f"per step: sequence 0, first {tokens} tokens, 1 KV head x {rr['pairs']} query "
              f"heads; oracle quantize then decode")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (dec + qt) / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(cfg),
        "quantize": {"value": rr["vectors"] * args.steps / qt / 1e6, "unit": "Mvec/s"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "kind": "oracle",
                         "cores": min(rr["threads"], rr["pairs"]), "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(cfg):
    return {"workload": cfg.name, "description": cfg.description, "n_seqs": cfg.n_seqs,
            "context": cfg.decode_lens()[0] if cfg.fixed_len else "varied",
            "n_q_heads": cfg.n_q_heads, "n_kv_heads": cfg.n_kv_heads, "head_dim": cfg.d,
            "kv_dtype": str(cfg.in_dtype).replace("torch.", ""),
            "quantize_chunk_tokens": cfg.quant_chunk or None,
            "l2": "inputs larger than L2; L2 flushed before each decode"}


# ------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    import rotated_bit_kv_isoquant_b200 as iq
    import workloads as wl

    rank, world, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    stream = torch.cuda.current_stream(dev)
    params = iq.isoq_make_params(wl.PARAM_SEED, cfg.d, cfg.n_kv_heads)
    layout = wl.page_layout(cfg)
    cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, layout.n_pages, layout.page_table, device=dev)
    calls = wl.prefill_calls(cfg)
    inputs = []
    for s, start, count in calls:
        K, V = wl.kv_tokens(cfg, s, start, count, device=dev)
        sid = torch.full((count,), s, dtype=torch.int32, device=dev)
        pos = torch.arange(start, start + count, dtype=torch.int32, device=dev)
        inputs.append((K, V, sid, pos))
    app = wl.append_kv(cfg, device=dev)
    Q = wl.queries(cfg, device=dev)
    lens = cfg.decode_lens()
    max_len = max(lens)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = torch.empty((cfg.n_seqs, cfg.n_q_heads, cfg.d), dtype=torch.float32, device=dev)
    wsb = iq.isoq_decode_workspace_bytes(cfg.n_seqs, cfg.n_q_heads, cfg.n_kv_heads, cfg.d, max_len)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty((2 * l2 // 4,), dtype=torch.int32, device=dev)

    n_vec = 2 * cfg.n_kv_heads * sum(c for _, _, c in calls)
    n_vec += 2 * cfg.n_kv_heads * app[0].shape[0]
    packed = sum(lens) * cfg.n_kv_heads * 2 * (3 * cfg.d // 8 + 2)
    launches_per_step = len(calls) + (1 if app[0].shape[0] else 0) + 2

    def quantize_all():
        for K, V, sid, pos in inputs:
            iq.isoq_quantize_append(params, cache, K, V, sid, pos, stream=stream)
        if app[0].shape[0]:
            iq.isoq_quantize_append(params, cache, app[0], app[1], app[2], app[3], stream=stream)

    def decode():
        iq.isoq_decode_attention(params, cache, Q, sl, max_len, out, cfg.scale, ws, stream=stream)

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(e_q0, e_q1, e_d0, e_d1):
        e_q0.record(stream)
        quantize_all()
        e_q1.record(stream)
        flush.zero_()
        e_d0.record(stream)
        decode()
        e_d1.record(stream)

    for _ in range(args.warmup):
        step(ev(), ev(), ev(), ev())
    torch.cuda.synchronize()
    assert iq.isoq_get_status(cache) == 0, "device status bits set during warm-up"

    evs = [(ev(), ev(), ev(), ev()) for _ in range(args.steps)]
    t_start, t_end = ev(), ev()
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for e in evs:
            step(*e)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = rank_max(t_start.elapsed_time(t_end))
    q_ms = rank_max(sum(a.elapsed_time(b) for a, b, _, _ in evs))
    d_ms = rank_max(sum(c.elapsed_time(d) for _, _, c, d in evs))
    dec_launch_ms = d_ms / args.steps

    value = weak_scaling_rate(packed, args.steps, world, d_ms) / 1e9
    qval = weak_scaling_rate(n_vec, args.steps, world, q_ms) / 1e6
    peak, peak_kind = _peaks()
    dec_gbs_1 = packed / (dec_launch_ms / 1e3) / 1e9
    q_bytes = n_vec * (cfg.d * (4 if cfg.in_dtype == torch.float32 else 2) + 3 * cfg.d // 8 + 2)
    q_gbs_1 = q_bytes / (q_ms / args.steps / 1e3) / 1e9
    tr_dec = _ncu_traffic("decode", cfg.name)
    tr_q = _ncu_traffic("quantize", cfg.name)

    # ---- e2e: host inputs (pinned), H2D inside the timed region, D2H of the output ----
    e2e = None
    if not args.no_e2e:
        host = [(K.cpu().pin_memory(), V.cpu().pin_memory()) for K, V, _, _ in inputs]
        hq = Q.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(k.numel() * k.element_size() * 2 for k, _ in host) + hq.numel() * hq.element_size()
        d2h = hout.numel() * hout.element_size()

        # the host-to-device copies run on their own stream, chunk by chunk, so that chunk
        # i is quantized while chunk i+1 crosses the link; a step's copies start after the
        # previous step's work (its buffers are free then)
        copy_stream = torch.cuda.Stream(device=dev)

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            copy_stream.wait_event(start)
            ready = []
            with torch.cuda.stream(copy_stream):
                for (hk, hv), (K, V, _, _) in zip(host, inputs):
                    K.copy_(hk, non_blocking=True)
                    V.copy_(hv, non_blocking=True)
                    e = torch.cuda.Event()
                    e.record(copy_stream)
                    ready.append(e)
                Q.copy_(hq, non_blocking=True)
                q_ready = torch.cuda.Event()
                q_ready.record(copy_stream)
            for e, (K, V, sid, pos) in zip(ready, inputs):
                stream.wait_event(e)
                iq.isoq_quantize_append(params, cache, K, V, sid, pos, stream=stream)
            if app[0].shape[0]:
                iq.isoq_quantize_append(params, cache, app[0], app[1], app[2], app[3],
                                        stream=stream)
            stream.wait_event(q_ready)
            decode()
            hout.copy_(out, non_blocking=True)

        e2e_steps = args.e2e_steps or args.steps
        e2e_step()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = rank_max(a.elapsed_time(b))
        e2e = {"value": weak_scaling_rate(packed, e2e_steps, world, e_ms) / 1e9,
               "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": e2e_steps, "ms_per_step": e_ms / e2e_steps,
               "what": "packed-KV bytes decoded per step / step time with the step's K, V and "
                       "Q copied from pinned host memory (on a copy stream, overlapping the "
                       "quantize-append of the chunks already copied), decode and the output "
                       "copied back"}

    line = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DECODE_DTYPE, "data": "synthetic",
        "hbm_frac_of_spec": dec_gbs_1 / SPEC_HBM_GBS,
        "config": _config(cfg),
        "quantize": {"value": qval, "unit": "Mvec/s", "ms_per_step": q_ms / args.steps,
                     "roofline": {"bound": "hbm", "achieved": q_gbs_1, "peak": peak,
                                  "unit": "GB/s", "frac": q_gbs_1 / peak, "traffic": tr_q,
                                  "peak_kind": peak_kind}},
        "decode_ms": dec_launch_ms,
        "roofline": {"bound": "hbm", "achieved": dec_gbs_1, "peak": peak, "unit": "GB/s",
                     "frac": dec_gbs_1 / peak, "traffic": tr_dec, "peak_kind": peak_kind,
                     "kernel": "decode (split-K kernel + combine kernel, one call)",
                     "algorithmic_bytes_per_launch": packed},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if not args.no_next:
        line["multi_token"] = _bench_multi_token(args, cfg, params, cache, lens, flush, stream,
                                                 rank_max, packed, peak, peak_kind)
        line["context_parallel"] = _bench_context_parallel(
            args, cfg, params, cache, layout, lens, Q, flush, stream, rank_max, world, rank,
            packed, peak, peak_kind)
        line["fused"] = _bench_fused(cfg, params, cache, inputs, lens, flush, stream,
                                     rank_max, peak, peak_kind)
        if cfg.d == 128:
            line["formats"] = _bench_formats(cfg, layout, inputs, app, Q, lens, flush, stream,
                                             rank_max, peak, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if not args.no_configs and not args.seqs:
        line["configs"] = _bench_configs(
            args, cfg, {"decode_GBps": dec_gbs_1, "decode_ms": dec_launch_ms,
                        "quantize_Mvec_s": qval / world, "quantize_frac": q_gbs_1 / peak,
                        "packed_bytes": packed, "vectors": n_vec,
                        "oracle": line.get("cpu_baseline")},
            flush, stream, rank_max, peak, peak_kind, dev,
            oracle_ok=(rank == 0 and world == 1 and not args.no_cpu_baseline))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def _time_calls(fn, flush, stream, iters: int = 5, warmup: int = 2) -> float:
    """Mean device time (ms) of fn() on `stream`, L2 flushed before every call."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(iters):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    return total / iters


def _bench_multi_token(args, cfg, params, cache, lens, flush, stream, rank_max, packed, peak,
                       peak_kind):
    """Causal attention of a chunk of query tokens per sequence on the same packed cache."""
    import torch

    import rotated_bit_kv_isoquant_b200 as iq
    import workloads as wl
    n_q = args.chunk
    dev = cache.blocks.device
    Qc = wl.query_chunk(cfg, n_q, device=dev)
    out = torch.empty((cfg.n_seqs, n_q, cfg.n_q_heads, cfg.d), dtype=torch.float32, device=dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    nb = iq.isoq_multi_token_workspace_bytes(cfg.n_seqs, n_q, cfg.n_q_heads, cfg.n_kv_heads,
                                             cfg.d, max(lens))
    ws = torch.empty((nb,), dtype=torch.uint8, device=dev)
    fn = lambda: iq.isoq_multi_token_attention(params, cache, Qc, sl, max(lens), out, cfg.scale,
                                               ws, stream=stream)
    ms = rank_max(_time_calls(fn, flush, stream))
    gbs = packed / (ms / 1e3) / 1e9
    # algorithmic work: scores and the value sum, 2 * 2 * d flops per (row, attended token)
    attended = sum(max(0, L - n_q + 1 + i) for L in lens for i in range(n_q))
    flops = 4.0 * cfg.d * cfg.n_q_heads * attended
    tf = flops / (ms / 1e3) / 1e12
    tpk, tpk_kind = _tensor_peak()
    return {"n_q": n_q, "ms_per_call": ms,
            "query_tokens_per_s": cfg.n_seqs * n_q / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": tpk, "unit": "TFLOP/s",
                         "frac": tf / tpk, "peak_kind": tpk_kind,
                         "flops_per_call": flops,
                         "note": "f16 products on tcgen05 (the query's high and low f16 parts "
                                 "double the score products, not counted)"},
            "hbm_view": {"achieved": gbs, "unit": "GB/s", "frac": gbs / peak,
                         "peak_kind": peak_kind,
                         "note": "packed KV read once per 128 rows of a KV head"}}


def _bench_fused(cfg, params, cache, inputs, lens, flush, stream, rank_max, peak, peak_kind):
    """Fused epilogues: the prefill quantize-append with RoPE applied to K in the kernel
    (pre-RoPE keys in, same cache), and one decode step's appends (one token per sequence)
    into 32 layers' caches as 32 calls versus one layer-batched call."""
    import torch

    import rotated_bit_kv_isoquant_b200 as iq
    import workloads as wl
    dev = cache.blocks.device
    tab = iq.isoq_rope_table(cfg.d, max(lens) + 1, device=dev)

    def quantize_rope():
        for K, V, sid, pos in inputs:
            iq.isoq_quantize_append_rope(params, cache, K, V, sid, pos, tab, stream=stream)

    n_vec = 2 * cfg.n_kv_heads * sum(K.shape[0] for K, _, _, _ in inputs)
    rope_ms = rank_max(_time_calls(quantize_rope, flush, stream, iters=2, warmup=1))
    n_layers = 32
    pt = torch.arange(cfg.n_seqs, dtype=torch.int32).reshape(cfg.n_seqs, 1)
    ps = [iq.isoq_make_params(wl.PARAM_SEED + l, cfg.d, cfg.n_kv_heads) for l in range(n_layers)]
    cs = [iq.PagedCache(cfg.d, cfg.n_kv_heads, cfg.n_seqs, pt, device=dev) for _ in range(n_layers)]
    g = torch.Generator(device=dev).manual_seed(3)
    Ks = [torch.randn((cfg.n_seqs, cfg.n_kv_heads, cfg.d), generator=g, device=dev).to(cfg.in_dtype)
          for _ in range(n_layers)]
    Vs = [torch.randn_like(k, dtype=torch.float32).to(cfg.in_dtype) for k in Ks]
    sid = torch.arange(cfg.n_seqs, dtype=torch.int32, device=dev)
    pos = torch.full((cfg.n_seqs,), 5, dtype=torch.int32, device=dev)
    step_tab = iq.isoq_rope_table(cfg.d, 64, device=dev)

    def per_layer():
        for l in range(n_layers):
            iq.isoq_quantize_append_rope(ps[l], cs[l], Ks[l], Vs[l], sid, pos, step_tab,
                                         stream=stream)

    def batched():
        iq.isoq_quantize_append_layers(ps, cs, Ks, Vs, sid, pos, rope_table=step_tab,
                                       stream=stream)

    t_sep = rank_max(_time_calls(per_layer, flush, stream, iters=20, warmup=3))
    t_bat = rank_max(_time_calls(batched, flush, stream, iters=20, warmup=3))
    return {"rope_quantize_Mvec_s": n_vec / (rope_ms / 1e3) / 1e6,
            "rope_quantize_ms": rope_ms,
            "decode_step_append_32_layers_us": {"per_layer_calls": t_sep * 1e3,
                                                "one_batched_call": t_bat * 1e3},
            "what": "RoPE applied to pre-RoPE K inside quantize-append (same cache and tokens as "
                    "the step); a decode step's 1-token-per-sequence appends into 32 layers"}


def _bench_formats(cfg, layout, inputs, app, Q, lens, flush, stream, rank_max, peak,
                   peak_kind):
    """The format variants on the same workload: quantize-append of the whole prefill and
    one decode per (bits, rotation), each with its own cache."""
    import torch

    import rotated_bit_kv_isoquant_b200 as iq
    import workloads as wl
    dev = Q.device
    res = {}
    for bits, rot in ((2, 0), (4, 0), (3, 1), (2, 1), (4, 1)):
        params = iq.isoq_make_params(wl.PARAM_SEED, cfg.d, cfg.n_kv_heads, bits=bits, rotation=rot)
        cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, layout.n_pages, layout.page_table, device=dev,
                              bits=bits)

        def quantize_all():
            for K, V, sid, pos in inputs:
                iq.isoq_quantize_append(params, cache, K, V, sid, pos, stream=stream)
            if app[0].shape[0]:
                iq.isoq_quantize_append(params, cache, app[0], app[1], app[2], app[3],
                                        stream=stream)

        q_ms = rank_max(_time_calls(quantize_all, flush, stream, iters=2, warmup=1))
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        out = torch.empty((cfg.n_seqs, cfg.n_q_heads, cfg.d), dtype=torch.float32, device=dev)
        nb = iq.isoq_decode_workspace_bytes(cfg.n_seqs, cfg.n_q_heads, cfg.n_kv_heads, cfg.d,
                                            max(lens))
        ws = torch.empty((nb,), dtype=torch.uint8, device=dev)
        fn = lambda: iq.isoq_decode_attention(params, cache, Q, sl, max(lens), out, cfg.scale, ws,
                                              stream=stream)
        d_ms = rank_max(_time_calls(fn, flush, stream))
        packed = sum(lens) * cfg.n_kv_heads * 2 * (bits * cfg.d // 8 + 2)
        n_vec = 2 * cfg.n_kv_heads * (sum(c for _, _, c in wl.prefill_calls(cfg)) + app[0].shape[0])
        q_bytes = n_vec * (cfg.d * (4 if cfg.in_dtype == torch.float32 else 2) + bits * cfg.d // 8 + 2)
        gbs = packed / (d_ms / 1e3) / 1e9
        res[f"{bits}bit_{'so2' if rot else 'so4'}"] = {
            "decode_GBps": gbs, "decode_frac": gbs / peak, "decode_ms": d_ms,
            "quantize_Mvec_s": n_vec / (q_ms / 1e3) / 1e6,
            "quantize_frac": q_bytes / (q_ms / 1e3) / 1e9 / peak,
            "packed_bytes_per_decode": packed}
        del cache, params
        torch.cuda.empty_cache()
    res["peak_kind"] = peak_kind
    return res


def _bench_context_parallel(args, cfg, params, cache, layout, lens, Q, flush, stream, rank_max,
                            world, rank, packed, peak, peak_kind):
    """One decode step of the whole workload with every context split over the ranks:
    each rank decodes its slice (a view of its replica's cache), one all-gather of the
    states, then the merge (strong scaling over the context)."""
    import torch

    from rotated_bit_kv_isoquant_b200.context_parallel import ContextParallelDecoder, slice_of
    view, local = slice_of(cache, layout.page_table, lens, world, rank)
    dec = ContextParallelDecoder(params, view, cfg.n_seqs, cfg.n_q_heads, max(1, max(local)))
    dev = cache.blocks.device
    sl = torch.tensor(local, dtype=torch.int32, device=dev)
    out = torch.empty((cfg.n_seqs, cfg.n_q_heads, cfg.d), dtype=torch.float32, device=dev)
    fn = lambda: dec(Q, sl, out, cfg.scale, stream=stream)
    ms = rank_max(_time_calls(fn, flush, stream))
    gbs = packed / (ms / 1e3) / 1e9
    return {"value": gbs, "unit": "GB/s", "scaling": "strong", "ms_per_call": ms,
            "n_gpus": world, "state_bytes_per_rank": int(dec.state.numel() * 4),
            "roofline_frac_per_gpu": gbs / world / peak, "peak_kind": peak_kind}


def _bench_configs(args, head_cfg, head, flush, stream, rank_max, peak, peak_kind, dev,
                   oracle_ok: bool):
    """Every workload of the configuration list on this GPU: the prefill quantised in its
    chunked calls (Mvec/s), the appended tokens, one decode step of every sequence (mean of
    10 calls, L2 flushed before each), the fraction of the measured and of the specified
    HBM peak, and the oracle on a bounded sample of the same workload.  The headline
    workload's numbers are the main measurement's."""
    import torch

    import rotated_bit_kv_isoquant_b200 as iq
    import workloads as wl
    res = {}
    for idx in range(1, len(wl.WORKLOADS) + 1):
        cfg = wl.workload(idx)
        lens = cfg.decode_lens()
        packed = sum(lens) * cfg.n_kv_heads * 2 * (3 * cfg.d // 8 + 2)
        in_b = 4 if cfg.in_dtype == torch.float32 else 2
        vec_bytes = cfg.d * in_b + 3 * cfg.d // 8 + 2
        if idx == head_cfg.idx:
            r = {"decode_GBps": head["decode_GBps"], "decode_ms": head["decode_ms"],
                 "quantize_Mvec_s": head["quantize_Mvec_s"],
                 "quantize_frac_measured": head["quantize_frac"],
                 "packed_bytes": head["packed_bytes"], "quantize_vectors": head["vectors"],
                 "oracle": head["oracle"], "source": "the main measurement"}
        else:
            params = iq.isoq_make_params(wl.PARAM_SEED, cfg.d, cfg.n_kv_heads)
            layout = wl.page_layout(cfg)
            cache = iq.PagedCache(cfg.d, cfg.n_kv_heads, layout.n_pages, layout.page_table,
                                  device=dev)
            q_ms, n_vec = 0.0, 0
            for s, start, count in wl.prefill_calls(cfg):
                K, V = wl.kv_tokens(cfg, s, start, count, device=dev)
                sid = torch.full((count,), s, dtype=torch.int32, device=dev)
                pos = torch.arange(start, start + count, dtype=torch.int32, device=dev)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                iq.isoq_quantize_append(params, cache, K, V, sid, pos, stream=stream)
                b.record(stream)
                torch.cuda.synchronize()
                q_ms += a.elapsed_time(b)
                n_vec += 2 * cfg.n_kv_heads * count
                del K, V
            app = wl.append_kv(cfg, device=dev)
            app_us = None
            if app[0].shape[0]:
                fn_app = lambda: iq.isoq_quantize_append(params, cache, *app, stream=stream)
                app_us = rank_max(_time_calls(fn_app, flush, stream, iters=10)) * 1e3
            Q = wl.queries(cfg, device=dev)
            sl = torch.tensor(lens, dtype=torch.int32, device=dev)
            out = torch.empty((cfg.n_seqs, cfg.n_q_heads, cfg.d), dtype=torch.float32, device=dev)
            nb = iq.isoq_decode_workspace_bytes(cfg.n_seqs, cfg.n_q_heads, cfg.n_kv_heads,
                                                cfg.d, max(lens))
            ws = torch.empty((max(nb, 16),), dtype=torch.uint8, device=dev)
            fn = lambda: iq.isoq_decode_attention(params, cache, Q, sl, max(lens), out,
                                                  cfg.scale, ws, stream=stream)
            d_ms = rank_max(_time_calls(fn, flush, stream, iters=10, warmup=3))
            assert iq.isoq_get_status(cache) == 0, f"status bits set on workload {idx}"
            q_ms = rank_max(q_ms)
            r = {"decode_GBps": packed / (d_ms / 1e3) / 1e9, "decode_ms": d_ms,
                 "quantize_Mvec_s": n_vec / (q_ms / 1e3) / 1e6,
                 "quantize_frac_measured": n_vec * vec_bytes / (q_ms / 1e3) / 1e9 / peak,
                 "packed_bytes": packed, "quantize_vectors": n_vec,
                 "decode_splits": iq.isoq_decode_num_splits(cfg.n_seqs, cfg.n_q_heads,
                                                            cfg.n_kv_heads, cfg.d, max(lens))}
            if app_us is not None:
                r["append_us"] = app_us
                r["append_vectors"] = 2 * cfg.n_kv_heads * app[0].shape[0]
            r["oracle"] = cpu_baseline(cfg, budget_s=2.5, single_core_s=1.5) if oracle_ok else None
            del cache, params, Q, out, ws
            torch.cuda.empty_cache()
        r["decode_frac_measured"] = r["decode_GBps"] / peak
        r["decode_frac_spec"] = r["decode_GBps"] / SPEC_HBM_GBS
        r["context"] = max(lens)
        r["target_applies"] = max(lens) >= 32768     # >= 0.70 of the HBM peak at 32k+ contexts
        res[cfg.name] = r
    res["peak"] = {"measured_GBps": peak, "kind": peak_kind, "spec_GBps": SPEC_HBM_GBS}
    return res


def main():
    args = _args()
    import workloads as wl
    cfg = wl.workload(args.config)
    if args.seqs:
        from dataclasses import replace
        cfg = replace(cfg, n_seqs=args.seqs)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
