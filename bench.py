#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

A step is one prefill call over the causal GQA workload (batch 4, 32 query /
8 key-value heads, 2048 tokens, head_dim 128, bf16, seed 1). The headline
``value`` is its throughput in TFLOP/s of algorithmic work (4 * head_dim per
visible query-key pair and query head). The same JSON line also carries the
paged split-KV decode workload (batch 64, lengths U[1024, 32768], 32/8 heads)
timed the same way, in GB/s of algorithmic KV traffic (also on an FP8 E4M3
copy of the cache, one scale per tensor), and the mixed batch
(8 prefill chunks of 512 queries on cached context plus 128 decode rows over
one paged cache) as a fraction of the combined tensor + HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own full batch (weak scaling, no
collective on the data path) and rank 0 prints one JSON line with the
max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import functools
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_tiled_exact_b200 import workloads as wl  # noqa: E402

METRIC = "attention TFLOP/s (prefill) & KV GB/s (decode), % of B200 roofline"
PREFILL_CFG = wl.CAUSAL_GQA_2K
DECODE_CFG = wl.PAGED_DECODE
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "prefill": ["attention_tiled_exact_b200/csrc/prefill_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh"],
    "decode": ["attention_tiled_exact_b200/csrc/decode_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh"],
    "decode_fp8": ["attention_tiled_exact_b200/csrc/decode_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh"],
}


def kernel_hash(kind: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kind: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", f"{kind}_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_sha") != kernel_hash(kind):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.rows.append([x.strip() for x in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------
# workloads on the device
# ----------------------------------------------------------------------------


def _dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def prefill_inputs(rank: int):
    import dataclasses
    cfg = dataclasses.replace(PREFILL_CFG, seed=PREFILL_CFG.seed + 1000 * rank)
    d = wl.make_prefill(cfg)
    flops = 4.0 * cfg.head_dim * cfg.batch * cfg.q_heads * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    return cfg, d, flops


@functools.lru_cache(maxsize=2)
def decode_inputs(rank: int, batch: int = 0):
    import dataclasses
    cfg = dataclasses.replace(DECODE_CFG, seed=DECODE_CFG.seed + 1000 * rank,
                              batch=batch if batch > 0 else DECODE_CFG.batch)
    d = wl.make_decode(cfg)
    total_tokens = int(d["kv_lens"].sum())
    kv_bytes = total_tokens * cfg.kv_heads * cfg.head_dim * 2 * 2
    io_bytes = cfg.batch * cfg.q_heads * (cfg.head_dim * 2 * 2 + 4)
    return cfg, d, float(kv_bytes + io_bytes)


def time_loop(fn, steps, warmup, world):
    """CUDA-event time of `steps` back-to-back calls after `warmup` calls (ms per step, max over ranks)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(stop) / steps
    return max_over_ranks(ms, world)


def run_ours(args, rank, world, local):
    import torch

    from attention_tiled_exact_b200 import binding as attn
    peaks, peak_src = load_peaks()

    result = {}
    if args.only in (None, "prefill"):
        result.update(bench_prefill(args, rank, world, local, attn, peaks, peak_src))
    if args.only in (None, "decode"):
        result["decode"] = bench_decode(args, rank, world, local, attn, peaks, peak_src)
    if args.only in (None, "decodefp8"):
        result["decode_fp8"] = bench_decode_fp8(args, rank, world, local, attn, peaks, peak_src)
    if args.only in (None, "mixed"):
        result["mixed"] = bench_mixed(args, rank, world, local, attn, peaks, peak_src)
    if args.only in (None, "prefill16k"):
        result["prefill_16k"] = bench_prefill_16k(args, rank, world, local, attn, peaks, peak_src)
    if args.only in (None, "sharedprefix"):
        result["shared_prefix"] = bench_shared_prefix(args, rank, world, local, attn, peaks, peak_src)
    if args.only in (None, "backward"):
        result["backward"] = bench_backward(args, rank, world, local, attn, peaks, peak_src)
    if args.only is not None:
        result["partial"] = f"--only {args.only}: profiling run, not a bench line"
    if rank == 0 and args.only is None:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return result


def bench_prefill(args, rank, world, local, attn, peaks, peak_src):
    import torch
    cfg, d, flops = prefill_inputs(rank)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")

    def prefill_step():
        attn.prefill(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse)

    with ClockSampler(local) as clk:
        ms = time_loop(prefill_step, args.steps, args.warmup, world)
    clocks = clk.summary()
    tflops = flops * world / (ms * 1e-3) / 1e12
    per_rank_tflops = flops / (ms * 1e-3) / 1e12
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])

    # e2e through the public call with host buffers: H2D inputs, prefill, D2H output + LSE
    hq = torch.from_numpy(d["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(d["v"].view(np.int16)).view(torch.bfloat16).pin_memory()
    ho = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        attn.prefill(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    if args.only is None:
        e2e_steps = max(3, min(args.steps, 10))
        ms_e2e = time_loop(e2e_step, e2e_steps, 2, world)
    else:
        ms_e2e = float("nan")
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = ho.numel() * 2 + hl.numel() * 4
    del hq, hk, hv, ho, hl

    result = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, per-rank seeds)",
        "config": {"workload": cfg.name, "batch": cfg.batch, "q_heads": cfg.q_heads, "kv_heads": cfg.kv_heads,
                   "seq_len": cfg.seqlen_q, "head_dim": cfg.head_dim, "causal": cfg.causal,
                   "parallelism": f"replicas x{world} (no collective)",
                   "l2": "inputs larger than L2 (Q 64 MiB + K/V 32 MiB + O 64 MiB per step)"},
        "roofline": {"bound": "tensor", "kernel": "prefill_fwd_kernel<128,2,false>",
                     "achieved": round(per_rank_tflops, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(per_rank_tflops / peak_t, 4),
                     "peak_source": f"{peak_src} bf16 burst (cuBLAS 8192^3)",
                     "frac_of_sustained": round(per_rank_tflops / peaks.get("bf16_tflops_sustained", 1400.0), 4),
                     "traffic": profiled_traffic("prefill"),
                     "algorithmic_flops_per_launch": flops},
        "e2e": {"value": round(flops * world / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    return result


def bench_decode(args, rank, world, local, attn, peaks, peak_src):
    import torch
    dcfg, dd, dbytes = decode_inputs(rank, args.decode_batch)
    dq = _dev_bf16(dd["q"])
    kc, vc = _dev_bf16(dd["k_pool"]), _dev_bf16(dd["v_pool"])
    bt = torch.from_numpy(dd["block_table"]).cuda()
    sl = torch.from_numpy(dd["kv_lens"]).cuda()
    max_len = int(dd["kv_lens"].max())
    dout = torch.empty_like(dq)
    dlse = torch.empty(dq.shape[:2], dtype=torch.float32, device="cuda")
    ws_bytes = attn.decode_workspace_bytes(dq, kc, vc, bt, sl, max_seq_len=max_len)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")

    def decode_step():
        attn.decode_paged(dq, kc, vc, bt, sl, dcfg.scale, max_seq_len=max_len, out=dout, lse=dlse, workspace=ws)

    dsteps = max(args.steps, 5)
    with ClockSampler(local) as dclk:
        dms = time_loop(decode_step, dsteps, args.warmup, world)
    peak_h = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    dgbs = dbytes * world / (dms * 1e-3) / 1e9
    per_rank_gbs = dbytes / (dms * 1e-3) / 1e9

    return {"workload": dcfg.name, "value": round(dgbs, 1), "unit": "GB/s", "ms_per_step": round(dms, 4),
            "steps": dsteps, "kv_tokens": int(dd["kv_lens"].sum()),
            "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<4>", "achieved": round(per_rank_gbs, 1),
                         "peak": peak_h, "unit": "GB/s", "frac": round(per_rank_gbs / peak_h, 4),
                         "peak_source": f"{peak_src} copy bandwidth", "traffic": profiled_traffic("decode"),
                         "algorithmic_bytes_per_launch": dbytes},
            "gpu_launches_per_step": 2, "clocks": dclk.summary()}


def bench_decode_fp8(args, rank, world, local, attn, peaks, peak_src):
    """The decode workload on an FP8 E4M3 cache (the bf16 pools quantised with one scale per tensor)."""
    import torch
    dcfg, dd, _ = decode_inputs(rank, args.decode_batch)
    kq, k_scale = wl.bf16_pool_to_e4m3(dd["k_pool"])
    vq, v_scale = wl.bf16_pool_to_e4m3(dd["v_pool"])
    tokens = int(dd["kv_lens"].sum())
    dbytes = float(tokens * dcfg.kv_heads * dcfg.head_dim * 1 * 2 + dcfg.batch * dcfg.q_heads * (dcfg.head_dim * 2 * 2 + 4))
    dq = _dev_bf16(dd["q"])
    kc, vc = torch.from_numpy(kq).cuda(), torch.from_numpy(vq).cuda()
    del kq, vq
    bt = torch.from_numpy(dd["block_table"]).cuda()
    sl = torch.from_numpy(dd["kv_lens"]).cuda()
    max_len = int(dd["kv_lens"].max())
    dout = torch.empty_like(dq)
    dlse = torch.empty(dq.shape[:2], dtype=torch.float32, device="cuda")
    ws = torch.empty(max(attn.decode_workspace_bytes(dq, kc, vc, bt, sl, max_seq_len=max_len), 1),
                     dtype=torch.uint8, device="cuda")

    def step():
        attn.decode_paged(dq, kc, vc, bt, sl, dcfg.scale, max_seq_len=max_len, out=dout, lse=dlse, workspace=ws,
                          k_scale=k_scale, v_scale=v_scale)

    dsteps = max(args.steps, 5)
    with ClockSampler(local) as clk:
        ms = time_loop(step, dsteps, args.warmup, world)
    peak_h = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    per_rank_gbs = dbytes / (ms * 1e-3) / 1e9
    return {"workload": dcfg.name + "_fp8_e4m3", "value": round(per_rank_gbs * world, 1), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "steps": dsteps, "kv_tokens": tokens,
            "kv_tokens_per_s": round(tokens * world / (ms * 1e-3), 1),
            "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<4,true>", "achieved": round(per_rank_gbs, 1),
                         "peak": peak_h, "unit": "GB/s", "frac": round(per_rank_gbs / peak_h, 4),
                         "peak_source": f"{peak_src} copy bandwidth", "traffic": profiled_traffic("decode_fp8"),
                         "algorithmic_bytes_per_launch": dbytes},
            "gpu_launches_per_step": 2, "clocks": clk.summary()}


def bench_shared_prefix(args, rank, world, local, attn, peaks, peak_src):
    """Decode of 64 sequences that share an 8192-token prefix (its blocks aliased
    in every table row) plus 64..2048 tokens of their own: the shared-prefix
    call against the plain decode over the same tables."""
    import dataclasses

    import torch
    cfg = dataclasses.replace(wl.SHARED_PREFIX_DECODE, seed=wl.SHARED_PREFIX_DECODE.seed + 1000 * rank)
    d = wl.make_shared_prefix_decode(cfg)
    q = _dev_bf16(d["q"])
    kc, vc = _dev_bf16(d["k_pool"]), _dev_bf16(d["v_pool"])
    bt = torch.from_numpy(d["block_table"]).cuda()
    sl = torch.from_numpy(d["kv_lens"]).cuda()
    max_len = int(d["kv_lens"].max())
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    ws_c = torch.empty(attn.decode_shared_prefix_workspace_bytes(q, kc, vc, bt, sl, cfg.prefix_len,
                                                                 max_seq_len=max_len), dtype=torch.uint8,
                       device="cuda")
    ws_p = torch.empty(max(attn.decode_workspace_bytes(q, kc, vc, bt, sl, max_seq_len=max_len), 1),
                       dtype=torch.uint8, device="cuda")

    def cascade():
        attn.decode_paged_shared_prefix(q, kc, vc, bt, sl, cfg.prefix_len, cfg.scale, max_seq_len=max_len,
                                        out=out, lse=lse, workspace=ws_c)

    def plain():
        attn.decode_paged(q, kc, vc, bt, sl, cfg.scale, max_seq_len=max_len, out=out, lse=lse, workspace=ws_p)

    steps = max(args.steps, 10)
    with ClockSampler(local) as clk:
        ms = time_loop(cascade, steps, args.warmup, world)
    ms_plain = time_loop(plain, steps, args.warmup, world)
    logical = int(d["kv_lens"].sum())                       # keys attended, summed over sequences
    unique = cfg.prefix_len + int(d["suffix_lens"].sum())   # distinct cached tokens
    ubytes = float(unique * cfg.kv_heads * cfg.head_dim * 2 * 2 + cfg.batch * cfg.q_heads * (cfg.head_dim * 4 + 4))
    prefix_flops = 4.0 * cfg.batch * cfg.q_heads * cfg.prefix_len * cfg.head_dim
    peak_h = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = ubytes / (ms * 1e-3) / 1e9
    max_splits = -(-(max_len - cfg.prefix_len) // 512)
    return {"workload": cfg.name, "value": round(logical * world / (ms * 1e-3), 1), "unit": "kv_tokens/s",
            "ms_per_step": round(ms, 4), "steps": steps, "kv_tokens": logical, "unique_kv_tokens": unique,
            "plain_decode_ms_per_step": round(ms_plain, 4), "speedup_vs_plain_decode": round(ms_plain / ms, 3),
            "roofline": {"bound": "hbm", "kernel": "whole call (prefix prefill + suffix decode + merge)",
                         "achieved": round(gbs, 1), "peak": peak_h, "unit": "GB/s", "frac": round(gbs / peak_h, 4),
                         "peak_source": f"{peak_src} copy bandwidth", "traffic": None,
                         "algorithmic_bytes_per_launch": ubytes, "prefix_tensor_flops": prefix_flops},
            "gpu_launches_per_step": 4 + (1 if max_splits > 1 else 0), "clocks": clk.summary()}


def bench_backward(args, rank, world, local, attn, peaks, peak_src):
    """Backward of the causal GQA prefill workload (4 x 32/8 heads x 2048 x 128):
    dQ, dK, dV from the library's own forward O (bf16) and LSE, bf16 gradients."""
    import torch
    cfg, d, fwd_flops = prefill_inputs(rank)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    do = _dev_bf16(wl.normal_bf16(cfg.seed + 1000 * rank, q.shape, 43))
    o, lse = attn.prefill(q, k, v, cfg.scale, cfg.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(2 * cfg.batch * cfg.q_heads * (-(-cfg.seqlen_q // 128) * 128) * 4 + 512, dtype=torch.uint8,
                     device="cuda")

    def step():
        attn.prefill_backward(q, k, v, o, lse, do, cfg.scale, cfg.causal, dq=dq, dk=dk, dv=dv, workspace=ws)

    steps = max(5, min(args.steps, 20))
    with ClockSampler(local) as clk:
        ms = time_loop(step, steps, args.warmup, world)
    flops = 2.5 * fwd_flops  # five products per visible pair (S, dP, dV, dK, dQ) against the forward's two
    tf = flops / (ms * 1e-3) / 1e12
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {"workload": cfg.name + "_backward", "value": round(tf * world, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "steps": steps,
            "roofline": {"bound": "tensor", "kernel": "whole call (prep + dK/dV + dQ)", "achieved": round(tf, 2),
                         "peak": peak_t, "unit": "TFLOP/s", "frac": round(tf / peak_t, 4),
                         "peak_source": f"{peak_src} bf16 GEMM", "algorithmic_flops_per_launch": flops,
                         "executed_flops_per_launch": 3.5 * fwd_flops},
            "gpu_launches_per_step": 3, "clocks": clk.summary()}


def bench_prefill_16k(args, rank, world, local, attn, peaks, peak_src):
    """Long-context causal GQA prefill: batch 1, 32/8 heads, 16384 tokens, head_dim 128."""
    import dataclasses

    import torch
    cfg = dataclasses.replace(wl.CAUSAL_GQA_16K, seed=wl.CAUSAL_GQA_16K.seed + 1000 * rank)
    d = wl.make_prefill(cfg)
    flops = 4.0 * cfg.head_dim * cfg.batch * cfg.q_heads * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    steps = max(5, min(args.steps, 20))
    with ClockSampler(local) as clk:
        ms = time_loop(lambda: attn.prefill(q, k, v, cfg.scale, True, out=o, lse=lse), steps, args.warmup, world)
    tf = flops / (ms * 1e-3) / 1e12
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {"workload": cfg.name, "value": round(tf * world, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "steps": steps, "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peak_t,
                                         "frac": round(tf / peak_t, 4), "algorithmic_flops_per_launch": flops},
            "gpu_launches_per_step": 1, "clocks": clk.summary()}


def bench_mixed(args, rank, world, local, attn, peaks, peak_src):
    """Chunked prefill of 8 x 512 queries on cached context + 128 decode rows, one pass."""
    import dataclasses

    import torch
    cfg = dataclasses.replace(wl.MIXED, seed=wl.MIXED.seed + 1000 * rank)
    d = wl.make_mixed(cfg)
    nc = cfg.chunks
    kc, vc = _dev_bf16(d["k_pool"]), _dev_bf16(d["v_pool"])
    table = torch.from_numpy(d["block_table"]).cuda()
    lens = torch.from_numpy(d["kv_lens"]).cuda()
    tp, lp = table[:nc].contiguous(), lens[:nc].contiguous()
    td, ld = table[nc:].contiguous(), lens[nc:].contiguous()
    qc, qd = _dev_bf16(d["q_chunk"]), _dev_bf16(d["q_dec"])
    oc = torch.empty_like(qc)
    lsec = torch.empty(qc.shape[:3], dtype=torch.float32, device="cuda")
    od = torch.empty_like(qd)
    lsed = torch.empty(qd.shape[:2], dtype=torch.float32, device="cuda")
    max_dec = int(d["kv_lens"][nc:].max())
    ws = torch.empty(max(1, attn.decode_workspace_bytes(qd, kc, vc, td, ld, max_seq_len=max_dec)),
                     dtype=torch.uint8, device="cuda")

    def step():
        attn.prefill_paged(qc, kc, vc, tp, lp, None, cfg.scale, True, out=oc, lse=lsec)
        attn.decode_paged(qd, kc, vc, td, ld, cfg.scale, max_seq_len=max_dec, out=od, lse=lsed, workspace=ws)

    steps = max(args.steps, 5)
    with ClockSampler(local) as clk:
        ms = time_loop(step, steps, args.warmup, world)
    flops = 4.0 * cfg.head_dim * cfg.q_heads * sum(
        wl.causal_pairs(cfg.chunk_len, int(k), True) for k in d["kv_lens"][:nc])
    dec_bytes = float(int(d["kv_lens"][nc:].sum()) * cfg.kv_heads * cfg.head_dim * 2 * 2 +
                      cfg.decodes * cfg.q_heads * (cfg.head_dim * 4 + 4))
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_h = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    ideal_ms = (flops / (peak_t * 1e12) + dec_bytes / (peak_h * 1e9)) * 1e3
    return {"workload": cfg.name, "ms_per_step": round(ms, 4), "steps": steps,
            "prefill_tflop": round(flops / 1e12, 4), "decode_gb": round(dec_bytes / 1e9, 3),
            "roofline": {"bound": "tensor+hbm", "ideal_ms": round(ideal_ms, 4), "frac": round(ideal_ms / ms, 4),
                         "peak_source": f"{peak_src}: {peak_t} TFLOP/s bf16, {peak_h} GB/s"},
            "gpu_launches_per_step": 3, "clocks": clk.summary()}


# ----------------------------------------------------------------------------
# the oracle on the host cores
# ----------------------------------------------------------------------------


def cpu_baseline(budget_s: float):
    """The fp64 oracle as it stands, on whole (batch, head) slices of the prefill workload."""
    from oracle import attention_ref as ref
    cfg = PREFILL_CFG
    d = wl.make_prefill(cfg)
    G = cfg.q_heads // cfg.kv_heads
    per_head = 4.0 * cfg.head_dim * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and done < cfg.batch * cfg.q_heads:
        b, h = divmod(done, cfg.q_heads)
        ref.attention_rows(d["q"][b, h], d["k"][b, h // G], d["v"][b, h // G], cfg.scale,
                           ref.causal_positions(cfg.seqlen_q, cfg.seqlen_k))
        done += 1
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max((x.get("num_threads", 1) for x in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count()
    return {"value": round(per_head * done / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} of {cfg.batch * cfg.q_heads} (batch, head) slices of {cfg.name}, fp64, "
                      f"materialised S, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    per_step_budget = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    from oracle import attention_ref as ref
    cfg = PREFILL_CFG
    d = wl.make_prefill(cfg)
    G = cfg.q_heads // cfg.kv_heads
    per_head = 4.0 * cfg.head_dim * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    pos = ref.causal_positions(cfg.seqlen_q, cfg.seqlen_k)

    def step():
        n, t0 = 0, time.perf_counter()
        while n == 0 or (time.perf_counter() - t0 < per_step_budget and n < cfg.batch * cfg.q_heads):
            b, h = divmod(n, cfg.q_heads)
            ref.attention_rows(d["q"][b, h], d["k"][b, h // G], d["v"][b, h // G], cfg.scale, pos)
            n += 1
        return n, time.perf_counter() - t0

    for _ in range(args.warmup):
        step()
    heads, secs = 0, 0.0
    for _ in range(args.steps):
        n, dt = step()
        heads += n
        secs += dt
    value = per_head * heads / secs / 1e12
    try:
        from threadpoolctl import threadpool_info
        threads = max((x.get("num_threads", 1) for x in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count()
    sample = (f"{heads} (batch, head) slices of {cfg.name} over {args.steps} steps "
              f"(about {per_step_budget:.1f} s each), fp64 oracle")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": cfg.name, "batch": cfg.batch, "q_heads": cfg.q_heads, "kv_heads": cfg.kv_heads,
                       "seq_len": cfg.seqlen_q, "head_dim": cfg.head_dim, "causal": cfg.causal},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "kind": "oracle", "cores": threads,
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only", choices=["prefill", "decode", "decodefp8", "mixed", "prefill16k", "sharedprefix", "backward"], default=None,
                    help="profiling aid: run one workload only (the line is then marked partial)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="profiling aid: fewer decode sequences (default: the full 64)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        res = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
