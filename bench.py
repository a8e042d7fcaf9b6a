#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

A step is one prefill call over the causal GQA workload (batch 4, 32 query /
8 key-value heads, 2048 tokens, head_dim 128, bf16, seed 1). The headline
``value`` is its throughput in TFLOP/s of algorithmic work (4 * head_dim per
visible query-key pair and query head). The same JSON line carries one object
per other workload, each timed the same way:

* ``tiny``: batch 1, 1 head, 128 x 128, head_dim 64, non-causal: the median
  latency of 200 individually timed calls;
* ``prefill_16k``: the long-context causal GQA prefill (1 x 32/8 x 16384);
* ``decode`` / ``decode_fp8``: the paged split-KV decode (64 sequences of
  U[1024, 32768] tokens, 32/8 heads), bf16 cache and an FP8 E4M3 copy, in GB/s
  of algorithmic KV traffic;
* ``mixed``: 8 prefill chunks of 512 queries on cached context plus 128 decode
  rows over one paged cache, as a fraction of the combined tensor + HBM
  roofline;
* ``shared_prefix``: decode of 64 sequences sharing an 8192-token prefix;
* ``backward``: dQ, dK, dV of the headline workload;
* ``decode_step_latency``: one small decode step (8 sequences) with the host
  in the loop: direct launch, CUDA-graph replay and persistent kernel.

On rank 0 of a 1-GPU run every workload also times the fp64 CPU oracle on a
bounded sample of the same inputs (``cpu_baseline``) and reports the largest
difference between the GPU outputs and the oracle on that sample
(``parity``: max|dO|, max|dLSE|).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 outside torchrun, bench.py starts the N ranks itself
(torch.distributed.run on 127.0.0.1). Every rank runs its own full batch
(weak scaling, no collective on the data path); rank 0 prints one JSON line
with the max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import functools
import hashlib
import json
import os
import socket
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
    "prefill": ["attention_tiled_exact_b200/csrc/prefill_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh",
                "attention_tiled_exact_b200/csrc/exp2_poly.cuh", "attention_tiled_exact_b200/csrc/bounds_check.cuh"],
    "prefill_16k": ["attention_tiled_exact_b200/csrc/prefill_sm100.cu",
                    "attention_tiled_exact_b200/csrc/sm100_ptx.cuh", "attention_tiled_exact_b200/csrc/exp2_poly.cuh",
                    "attention_tiled_exact_b200/csrc/bounds_check.cuh"],
    "decode": ["attention_tiled_exact_b200/csrc/decode_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh",
               "attention_tiled_exact_b200/csrc/bounds_check.cuh"],
    "decode_fp8": ["attention_tiled_exact_b200/csrc/decode_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh",
                   "attention_tiled_exact_b200/csrc/bounds_check.cuh"],
    "backward": ["attention_tiled_exact_b200/csrc/backward_sm100.cu", "attention_tiled_exact_b200/csrc/sm100_ptx.cuh",
                 "attention_tiled_exact_b200/csrc/bounds_check.cuh"],
}
LEGS = ("tiny", "prefill", "prefill16k", "decode", "decodefp8", "mixed", "sharedprefix", "backward", "decodesteps")


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


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_ranks(n: int, argv) -> int:
    """Run this script as n ranks under torch.distributed.run (127.0.0.1); returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.run(cmd).returncode


def dist_setup(n_gpus: int, need_cuda: bool = True):
    """Join the process group of a torchrun launch; returns (rank, world, local rank).

    The launch must have exactly n_gpus ranks. NCCL over the GPUs when CUDA is
    there, gloo on a CPU-only host (the host-logic checks)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"bench.py: --gpus {n_gpus} but the launch has {world} ranks")
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=300)
        if torch.cuda.is_available():
            if torch.cuda.device_count() < world:
                raise SystemExit(f"bench.py: {world} ranks but only {torch.cuda.device_count()} GPUs")
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        elif need_cuda:
            raise SystemExit("bench.py: no CUDA device")
        else:
            dist.init_process_group("gloo", timeout=timeout)
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
# timing
# ----------------------------------------------------------------------------


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


def time_repeats(fn, steps, world, min_total_ms=1000.0, max_brackets=400):
    """More brackets of `steps` back-to-back calls, until about `min_total_ms` of
    device time: ms per step of each bracket (max over ranks per bracket)."""
    out, total = [], 0.0
    while total < min_total_ms and len(out) < max_brackets:
        ms = time_loop(fn, steps, 0, world)
        out.append(ms)
        total += ms * steps
    return out


def latency_median(fn, n, warmup):
    """Median and percentiles of `n` individually timed calls (CUDA events around each, ms)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()  # one call at a time: the latency of a call, not the rate of a queue
    ts = sorted(a.elapsed_time(b) for a, b in evs)
    return {"median_ms": ts[n // 2], "p10_ms": ts[n // 10], "p90_ms": ts[(9 * n) // 10], "calls": n}


# ----------------------------------------------------------------------------
# the oracle on the host cores (rank 0, 1-GPU runs): throughput on a bounded
# sample of each workload and the GPU's largest deviation from it there
# ----------------------------------------------------------------------------


def blas_info():
    try:
        from threadpoolctl import threadpool_info
        info = [x for x in threadpool_info() if x.get("user_api") == "blas"]
        if info:
            return max(x.get("num_threads", 1) for x in info), ",".join(
                sorted({f"{x.get('internal_api')} {x.get('version')}" for x in info}))
    except Exception:
        pass
    return os.cpu_count(), "unknown"


def _cpu_record(value, unit, sample, seconds):
    threads, vendor = blas_info()
    return {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "blas": vendor,
            "sample": f"{sample}; {seconds:.1f} s of fp64 oracle work on the host cores"}


def _parity(o_gpu, o_ref, l_gpu, l_ref, rows, of_rows, out_dtype):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    l_gpu = np.asarray(l_gpu, dtype=np.float64)
    fin = np.isfinite(l_ref)
    same_inf = bool(np.array_equal(np.isneginf(l_gpu), np.isneginf(l_ref)))
    dl = float(np.abs(l_gpu[fin] - l_ref[fin]).max()) if fin.any() else 0.0
    return {"max_abs_dO": float(np.abs(o_gpu - o_ref).max()), "max_abs_dLSE": dl, "lse_inf_pattern_equal": same_inf,
            "rows_checked": int(rows), "of_rows": int(of_rows), "out_dtype": out_dtype}


def _bf16_to_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_prefill_slices(d, cfg, o_gpu, lse_gpu, budget_s, seed):
    """Whole (batch, head) slices in a seeded order until the budget is spent."""
    from oracle import attention_ref as ref
    G = cfg.q_heads // cfg.kv_heads
    pos = ref.causal_positions(cfg.seqlen_q, cfg.seqlen_k) if cfg.causal else None
    per_head = 4.0 * cfg.head_dim * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    order = np.random.default_rng(seed).permutation(cfg.batch * cfg.q_heads)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    t0, done = time.perf_counter(), 0
    while done < len(order) and (done == 0 or time.perf_counter() - t0 < budget_s):
        b, h = divmod(int(order[done]), cfg.q_heads)
        o, lse = ref.attention_rows(d["q"][b, h], d["k"][b, h // G], d["v"][b, h // G], cfg.scale, pos)
        ref_o.append(o), ref_l.append(lse)
        got_o.append(o_gpu[b, h]), got_l.append(lse_gpu[b, h])
        done += 1
    dt = time.perf_counter() - t0
    cpu = _cpu_record(round(per_head * done / dt / 1e12, 6), "TFLOP/s",
                      f"{done} of {len(order)} (batch, head) slices of {cfg.name}", dt)
    par = _parity(np.stack(got_o), np.stack(ref_o), np.stack(got_l), np.stack(ref_l), done * cfg.seqlen_q,
                  len(order) * cfg.seqlen_q, "bf16")
    return cpu, par


def oracle_prefill_row_chunks(d, cfg, o_rows_fn, lse_gpu, budget_s, seed, chunk=256):
    """Chunks of `chunk` query rows (all their keys) of seeded heads until the budget is spent."""
    from oracle import attention_ref as ref
    G = cfg.q_heads // cfg.kv_heads
    pos = ref.causal_positions(cfg.seqlen_q, cfg.seqlen_k)
    rng = np.random.default_rng(seed)
    n_chunks = cfg.seqlen_q // chunk
    got_o, ref_o, got_l, ref_l = [], [], [], []
    flops, rows = 0.0, 0
    t0 = time.perf_counter()
    while rows == 0 or time.perf_counter() - t0 < budget_s:
        b, h, c = int(rng.integers(cfg.batch)), int(rng.integers(cfg.q_heads)), int(rng.integers(n_chunks))
        r0, r1 = c * chunk, (c + 1) * chunk
        o, lse = ref.attention_rows(d["q"][b, h, r0:r1], d["k"][b, h // G], d["v"][b, h // G], cfg.scale,
                                    pos[r0:r1] if cfg.causal else None)
        ref_o.append(o), ref_l.append(lse)
        got_o.append(o_rows_fn(b, h, r0, r1)), got_l.append(lse_gpu[b, h, r0:r1])
        vis = np.clip(pos[r0:r1] + 1, 0, cfg.seqlen_k).sum() if cfg.causal else chunk * cfg.seqlen_k
        flops += 4.0 * cfg.head_dim * float(vis)
        rows += chunk
    dt = time.perf_counter() - t0
    cpu = _cpu_record(round(flops / dt / 1e12, 6), "TFLOP/s",
                      f"{rows // chunk} chunks of {chunk} query rows (all visible keys) of {cfg.name}", dt)
    par = _parity(np.concatenate(got_o), np.concatenate(ref_o), np.concatenate(got_l), np.concatenate(ref_l), rows,
                  cfg.batch * cfg.q_heads * cfg.seqlen_q, "bf16")
    return cpu, par


def oracle_decode_sequences(dd, o_gpu, lse_gpu, budget_s, seed, fp8_scales=None, bytes_per_elem=2,
                            unit="GB/s", out_dtype="bf16"):
    """Whole sequences (all query heads) in a seeded order until the budget is spent."""
    from oracle import attention_ref as ref
    B, Hq, D = dd["q"].shape
    Hkv = dd["k_pool"].shape[1]
    order = np.random.default_rng(seed).permutation(B)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    nbytes, tokens, done = 0.0, 0, 0
    t0 = time.perf_counter()
    while done < B and (done == 0 or time.perf_counter() - t0 < budget_s):
        b = int(order[done])
        rows = [(b, h) for h in range(Hq)]
        if fp8_scales is None:
            o, lse = ref.ref_decode_paged(dd["q"], dd["k_pool"], dd["v_pool"], dd["block_table"], dd["kv_lens"],
                                          dd["scale"], rows=rows)
        else:
            o, lse = ref.ref_decode_paged_fp8(dd["q"], dd["k_pool"], dd["v_pool"], fp8_scales[0], fp8_scales[1],
                                              dd["block_table"], dd["kv_lens"], dd["scale"], rows=rows)
        ref_o.append(o), ref_l.append(lse)
        got_o.append(o_gpu[b]), got_l.append(lse_gpu[b])
        L = int(dd["kv_lens"][b])
        nbytes += L * Hkv * D * bytes_per_elem * 2 + Hq * (D * 2 * 2 + 4)
        tokens += L
        done += 1
    dt = time.perf_counter() - t0
    value = tokens / dt if unit == "kv_tokens/s" else nbytes / dt / 1e9
    cpu = _cpu_record(round(value, 3), unit, f"{done} of {B} sequences ({tokens} cached tokens), all heads", dt)
    par = _parity(np.stack(got_o), np.stack(ref_o), np.stack(got_l), np.stack(ref_l), done * Hq, B * Hq, out_dtype)
    return cpu, par


# ----------------------------------------------------------------------------
# workloads on the device
# ----------------------------------------------------------------------------


def _dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _with_rank_seed(cfg, rank):
    import dataclasses
    return dataclasses.replace(cfg, seed=cfg.seed + 1000 * rank)


def prefill_inputs(rank: int):
    cfg = _with_rank_seed(PREFILL_CFG, rank)
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


class Ctx:
    """What every leg needs: the parsed arguments, the rank layout, the library and the peaks."""

    def __init__(self, args, rank, world, local, attn, peaks, peak_src):
        self.args, self.rank, self.world, self.local = args, rank, world, local
        self.attn, self.peaks, self.peak_src = attn, peaks, peak_src

    @property
    def with_oracle(self) -> bool:
        """The oracle legs run on rank 0 of a 1-GPU full run only."""
        return self.rank == 0 and self.world == 1 and self.args.only is None and self.args.cpu_seconds > 0

    def peak(self, key):
        return self.peaks.get(key, FALLBACK_PEAKS[key])


def bench_prefill(c: Ctx):
    import torch
    args, world, attn = c.args, c.world, c.attn
    cfg, d, flops = prefill_inputs(c.rank)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")

    def prefill_step():
        attn.prefill(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse)

    with ClockSampler(c.local) as clk:
        ms = time_loop(prefill_step, args.steps, args.warmup, world)
        reps = time_repeats(prefill_step, args.steps, world) if args.only is None else []
    clocks = clk.summary()
    tflops = flops * world / (ms * 1e-3) / 1e12
    per_rank_tflops = flops / (ms * 1e-3) / 1e12
    peak_t = c.peak("bf16_tflops")

    # e2e through the public host-buffer call: every step copies Q/K/V from
    # pinned host memory and O/LSE back, one batch entry per chunk, the copies
    # of one chunk overlapping the prefill of another (attn_prefill_from_host;
    # whole batch entries measured fastest: smaller chunks make smaller,
    # slower prefill launches); the timed region ends when O and LSE are in
    # host memory.
    hq = torch.from_numpy(d["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(d["v"].view(np.int16)).view(torch.bfloat16).pin_memory()
    ho = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        attn.prefill_from_host(hq, hk, hv, q, k, v, o, ho, lse, hl, cfg.scale, cfg.causal, kv_heads_per_chunk=0)

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
                     "peak_source": f"{c.peak_src} bf16 burst (cuBLAS 8192^3)",
                     "frac_of_sustained": round(per_rank_tflops / c.peak("bf16_tflops_sustained"), 4),
                     "traffic": profiled_traffic("prefill"),
                     "algorithmic_flops_per_launch": flops},
        "e2e": {"value": round(flops * world / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if reps:
        med = statistics.median(reps)
        result["repeats"] = {"brackets": len(reps), "steps_each": args.steps,
                             "median_ms_per_step": round(med, 4), "min_ms_per_step": round(min(reps), 4),
                             "max_ms_per_step": round(max(reps), 4),
                             "median_tflops": round(flops / (med * 1e-3) / 1e12, 2),
                             "median_frac": round(flops / (med * 1e-3) / 1e12 / peak_t, 4)}
        if clocks.get("sm_mhz"):
            result["repeats"]["kcycles_per_step_at_median_sm_clock"] = round(med * clocks["sm_mhz"], 1)
    if c.with_oracle:
        o_host, l_host = _bf16_to_f64(o), lse.cpu().numpy()
        cpu, par = oracle_prefill_slices(d, cfg, o_host, l_host, args.cpu_seconds, seed=11)
        result["cpu_baseline"] = cpu
        result["parity"] = {cfg.name: par}
    return result


def bench_tiny(c: Ctx):
    """The tiny non-causal problem (1 x 1 x 128 x 128 x 64): a latency figure."""
    import torch
    cfg = wl.TINY
    d = wl.make_prefill(cfg)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")

    def step():
        c.attn.prefill(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse)

    lat = latency_median(step, 200, c.args.warmup)
    flops = 4.0 * cfg.head_dim * cfg.seqlen_q * cfg.seqlen_k
    res = {"workload": cfg.name, "unit": "ms (median call latency)", "value": round(lat["median_ms"], 5),
           "latency": {k: (round(v, 5) if isinstance(v, float) else v) for k, v in lat.items()},
           "algorithmic_flops": flops, "roofline": {"bound": "latency", "frac": None,
                                                    "note": "one 128-row tile: no throughput roofline applies"},
           "gpu_launches_per_step": 1}
    if c.with_oracle:
        from oracle import attention_ref as ref
        t0 = time.perf_counter()
        O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], False)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = _cpu_record(round(dt * 1e3, 4), "ms per call", f"the whole of {cfg.name}", dt)
        res["parity"] = {cfg.name: _parity(_bf16_to_f64(o), O_ref, lse.cpu().numpy(), L_ref, cfg.seqlen_q,
                                           cfg.seqlen_q, "bf16")}
    return res


def bench_decode(c: Ctx):
    import torch
    args, world, attn = c.args, c.world, c.attn
    dcfg, dd, dbytes = decode_inputs(c.rank, args.decode_batch)
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
    with ClockSampler(c.local) as dclk:
        dms = time_loop(decode_step, dsteps, args.warmup, world)
    peak_h = c.peak("hbm_gbs")
    dgbs = dbytes * world / (dms * 1e-3) / 1e9
    per_rank_gbs = dbytes / (dms * 1e-3) / 1e9

    res = {"workload": dcfg.name, "value": round(dgbs, 1), "unit": "GB/s", "ms_per_step": round(dms, 4),
           "steps": dsteps, "kv_tokens": int(dd["kv_lens"].sum()),
           "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<4> + lse_combine_kernel (one step)",
                        "achieved": round(per_rank_gbs, 1), "peak": peak_h, "unit": "GB/s",
                        "frac": round(per_rank_gbs / peak_h, 4), "peak_source": f"{c.peak_src} copy bandwidth",
                        "traffic": profiled_traffic("decode"), "algorithmic_bytes_per_launch": dbytes},
           "gpu_launches_per_step": 2, "clocks": dclk.summary()}
    if c.with_oracle:
        cpu, par = oracle_decode_sequences(dd, _bf16_to_f64(dout), dlse.cpu().numpy(), args.cpu_seconds, seed=12)
        res["cpu_baseline"] = cpu
        res["parity"] = {dcfg.name: par}
    return res


def bench_decode_fp8(c: Ctx):
    """The decode workload on an FP8 E4M3 cache (the bf16 pools quantised with one scale per tensor)."""
    import torch
    args, world, attn = c.args, c.world, c.attn
    dcfg, dd, _ = decode_inputs(c.rank, args.decode_batch)
    kq, k_scale = wl.bf16_pool_to_e4m3(dd["k_pool"])
    vq, v_scale = wl.bf16_pool_to_e4m3(dd["v_pool"])
    tokens = int(dd["kv_lens"].sum())
    dbytes = float(tokens * dcfg.kv_heads * dcfg.head_dim * 1 * 2 + dcfg.batch * dcfg.q_heads * (dcfg.head_dim * 2 * 2 + 4))
    dq = _dev_bf16(dd["q"])
    kc, vc = torch.from_numpy(kq).cuda(), torch.from_numpy(vq).cuda()
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
    with ClockSampler(c.local) as clk:
        ms = time_loop(step, dsteps, args.warmup, world)
    peak_h = c.peak("hbm_gbs")
    per_rank_gbs = dbytes / (ms * 1e-3) / 1e9
    res = {"workload": dcfg.name + "_fp8_e4m3", "value": round(per_rank_gbs * world, 1), "unit": "GB/s",
           "ms_per_step": round(ms, 4), "steps": dsteps, "kv_tokens": tokens,
           "kv_tokens_per_s": round(tokens * world / (ms * 1e-3), 1),
           "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<4,true> + lse_combine_kernel (one step)",
                        "achieved": round(per_rank_gbs, 1), "peak": peak_h, "unit": "GB/s",
                        "frac": round(per_rank_gbs / peak_h, 4), "peak_source": f"{c.peak_src} copy bandwidth",
                        "traffic": profiled_traffic("decode_fp8"), "algorithmic_bytes_per_launch": dbytes},
           "gpu_launches_per_step": 2, "clocks": clk.summary()}
    if c.with_oracle:
        d8 = dict(dd, k_pool=kq, v_pool=vq)
        cpu, par = oracle_decode_sequences(d8, _bf16_to_f64(dout), dlse.cpu().numpy(), args.cpu_seconds, seed=13,
                                           fp8_scales=(k_scale, v_scale), bytes_per_elem=1)
        res["cpu_baseline"] = cpu
        res["parity"] = {dcfg.name + "_fp8_e4m3": par}
    return res


def bench_shared_prefix(c: Ctx):
    """Decode of 64 sequences that share an 8192-token prefix (its blocks aliased
    in every table row) plus 64..2048 tokens of their own: the shared-prefix
    call against the plain decode over the same tables."""
    import torch
    args, world, attn = c.args, c.world, c.attn
    cfg = _with_rank_seed(wl.SHARED_PREFIX_DECODE, c.rank)
    d = wl.make_shared_prefix_decode(cfg)
    q = _dev_bf16(d["q"])
    kc, vc = _dev_bf16(d["k_pool"]), _dev_bf16(d["v_pool"])
    bt = torch.from_numpy(d["block_table"]).cuda()
    sl = torch.from_numpy(d["kv_lens"]).cuda()
    max_len = int(d["kv_lens"].max())
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    out_p = torch.empty_like(q)
    lse_p = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    ws_c = torch.empty(attn.decode_shared_prefix_workspace_bytes(q, kc, vc, bt, sl, cfg.prefix_len,
                                                                 max_seq_len=max_len), dtype=torch.uint8,
                       device="cuda")
    ws_p = torch.empty(max(attn.decode_workspace_bytes(q, kc, vc, bt, sl, max_seq_len=max_len), 1),
                       dtype=torch.uint8, device="cuda")

    def cascade():
        attn.decode_paged_shared_prefix(q, kc, vc, bt, sl, cfg.prefix_len, cfg.scale, max_seq_len=max_len,
                                        out=out, lse=lse, workspace=ws_c)

    def plain():
        attn.decode_paged(q, kc, vc, bt, sl, cfg.scale, max_seq_len=max_len, out=out_p, lse=lse_p, workspace=ws_p)

    steps = max(args.steps, 10)
    with ClockSampler(c.local) as clk:
        ms = time_loop(cascade, steps, args.warmup, world)
    ms_plain = time_loop(plain, steps, args.warmup, world)
    logical = int(d["kv_lens"].sum())                       # keys attended, summed over sequences
    unique = cfg.prefix_len + int(d["suffix_lens"].sum())   # distinct cached tokens
    ubytes = float(unique * cfg.kv_heads * cfg.head_dim * 2 * 2 + cfg.batch * cfg.q_heads * (cfg.head_dim * 4 + 4))
    prefix_flops = 4.0 * cfg.batch * cfg.q_heads * cfg.prefix_len * cfg.head_dim
    peak_h = c.peak("hbm_gbs")
    gbs = ubytes / (ms * 1e-3) / 1e9
    res = {"workload": cfg.name, "value": round(logical * world / (ms * 1e-3), 1), "unit": "kv_tokens/s",
           "ms_per_step": round(ms, 4), "steps": steps, "kv_tokens": logical, "unique_kv_tokens": unique,
           "plain_decode_ms_per_step": round(ms_plain, 4), "speedup_vs_plain_decode": round(ms_plain / ms, 3),
           "roofline": {"bound": "hbm", "kernel": "whole call (prefix prefill + suffix decode + merge)",
                        "achieved": round(gbs, 1), "peak": peak_h, "unit": "GB/s", "frac": round(gbs / peak_h, 4),
                        "peak_source": f"{c.peak_src} copy bandwidth", "traffic": None,
                        "algorithmic_bytes_per_launch": ubytes, "prefix_tensor_flops": prefix_flops},
           "gpu_launches_per_step": 4, "clocks": clk.summary()}
    if c.with_oracle:
        cpu, par = oracle_decode_sequences(d, _bf16_to_f64(out), lse.cpu().numpy(), args.cpu_seconds, seed=14,
                                           unit="kv_tokens/s")
        res["cpu_baseline"] = cpu
        res["parity"] = {cfg.name: par}
    return res


def bench_backward(c: Ctx):
    """Backward of the causal GQA prefill workload (4 x 32/8 heads x 2048 x 128):
    dQ, dK, dV from the library's own forward O (bf16) and LSE, bf16 gradients."""
    import torch
    args, world, attn = c.args, c.world, c.attn
    cfg, d, fwd_flops = prefill_inputs(c.rank)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    do_bits = wl.normal_bf16(cfg.seed, q.shape, 43)
    do = _dev_bf16(do_bits)
    o, lse = attn.prefill(q, k, v, cfg.scale, cfg.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(2 * cfg.batch * cfg.q_heads * (-(-cfg.seqlen_q // 128) * 128) * 4 + 512, dtype=torch.uint8,
                     device="cuda")

    def step():
        attn.prefill_backward(q, k, v, o, lse, do, cfg.scale, cfg.causal, dq=dq, dk=dk, dv=dv, workspace=ws)

    steps = max(5, min(args.steps, 20))
    with ClockSampler(c.local) as clk:
        ms = time_loop(step, steps, args.warmup, world)
    flops = 2.5 * fwd_flops  # five products per visible pair (S, dP, dV, dK, dQ) against the forward's two
    tf = flops / (ms * 1e-3) / 1e12
    peak_t = c.peak("bf16_tflops")
    res = {"workload": cfg.name + "_backward", "value": round(tf * world, 2), "unit": "TFLOP/s",
           "ms_per_step": round(ms, 4), "steps": steps,
           "roofline": {"bound": "tensor", "kernel": "whole call (prep + dK/dV + dQ)", "achieved": round(tf, 2),
                        "peak": peak_t, "unit": "TFLOP/s", "frac": round(tf / peak_t, 4),
                        "peak_source": f"{c.peak_src} bf16 GEMM", "algorithmic_flops_per_launch": flops,
                        "executed_flops_per_launch": 3.5 * fwd_flops, "traffic": profiled_traffic("backward")},
           "gpu_launches_per_step": 3, "clocks": clk.summary()}
    if c.with_oracle:
        from oracle import attention_ref as ref
        G = cfg.q_heads // cfg.kv_heads
        order = np.random.default_rng(15).permutation(cfg.batch * cfg.kv_heads)
        g = {n: _bf16_to_f64(t) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
        worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
        t0, done = time.perf_counter(), 0
        while done < len(order) and (done == 0 or time.perf_counter() - t0 < args.cpu_seconds):
            b, kvh = divmod(int(order[done]), cfg.kv_heads)
            hs = slice(kvh * G, (kvh + 1) * G)
            r = ref.ref_attention_backward(d["q"][b:b + 1, hs], d["k"][b:b + 1, kvh:kvh + 1],
                                           d["v"][b:b + 1, kvh:kvh + 1], do_bits[b:b + 1, hs], cfg.scale, True)
            for n, got in (("dq", g["dq"][b:b + 1, hs]), ("dk", g["dk"][b:b + 1, kvh:kvh + 1]),
                           ("dv", g["dv"][b:b + 1, kvh:kvh + 1])):
                worst[n] = max(worst[n], float(np.abs(got - r[n]).max() / np.abs(r[n]).max()))
            done += 1
        dt = time.perf_counter() - t0
        per_group = 10.0 * cfg.head_dim * G * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, True)
        res["cpu_baseline"] = _cpu_record(round(per_group * done / dt / 1e12, 6), "TFLOP/s",
                                          f"{done} of {len(order)} (batch, kv head) groups", dt)
        res["parity"] = {cfg.name + "_backward": {
            "max_abs_err_over_max_abs_ref": {n: round(x, 6) for n, x in worst.items()}, "gate": 1e-2,
            "groups_checked": done, "of_groups": len(order), "grad_dtype": "bf16"}}
    return res


def bench_prefill_16k(c: Ctx):
    """Long-context causal GQA prefill: batch 1, 32/8 heads, 16384 tokens, head_dim 128."""
    import torch
    args, world, attn = c.args, c.world, c.attn
    cfg = _with_rank_seed(wl.CAUSAL_GQA_16K, c.rank)
    d = wl.make_prefill(cfg)
    flops = 4.0 * cfg.head_dim * cfg.batch * cfg.q_heads * wl.causal_pairs(cfg.seqlen_q, cfg.seqlen_k, cfg.causal)
    q, k, v = _dev_bf16(d["q"]), _dev_bf16(d["k"]), _dev_bf16(d["v"])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    steps = max(5, min(args.steps, 20))
    with ClockSampler(c.local) as clk:
        ms = time_loop(lambda: attn.prefill(q, k, v, cfg.scale, True, out=o, lse=lse), steps, args.warmup, world)
    tf = flops / (ms * 1e-3) / 1e12
    peak_t = c.peak("bf16_tflops")
    res = {"workload": cfg.name, "value": round(tf * world, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
           "steps": steps, "roofline": {"bound": "tensor", "kernel": "prefill_fwd_kernel<128,2,false>",
                                        "achieved": round(tf, 2), "peak": peak_t, "unit": "TFLOP/s",
                                        "frac": round(tf / peak_t, 4), "traffic": profiled_traffic("prefill_16k"),
                                        "algorithmic_flops_per_launch": flops},
           "gpu_launches_per_step": 1, "clocks": clk.summary()}
    if c.with_oracle:
        def o_rows(b, h, r0, r1):
            return o[b, h, r0:r1].to(torch.float64).cpu().numpy()
        cpu, par = oracle_prefill_row_chunks(d, cfg, o_rows, lse.cpu().numpy(), args.cpu_seconds, seed=16)
        res["cpu_baseline"] = cpu
        res["parity"] = {cfg.name: par}
    return res


def bench_mixed(c: Ctx):
    """Chunked prefill of 8 x 512 queries on cached context + 128 decode rows, one pass."""
    import torch
    args, world, attn = c.args, c.world, c.attn
    cfg = _with_rank_seed(wl.MIXED, c.rank)
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
    with ClockSampler(c.local) as clk:
        ms = time_loop(step, steps, args.warmup, world)
    flops = 4.0 * cfg.head_dim * cfg.q_heads * sum(
        wl.causal_pairs(cfg.chunk_len, int(k), True) for k in d["kv_lens"][:nc])
    dec_bytes = float(int(d["kv_lens"][nc:].sum()) * cfg.kv_heads * cfg.head_dim * 2 * 2 +
                      cfg.decodes * cfg.q_heads * (cfg.head_dim * 4 + 4))
    peak_t = c.peak("bf16_tflops")
    peak_h = c.peak("hbm_gbs")
    ideal_ms = (flops / (peak_t * 1e12) + dec_bytes / (peak_h * 1e9)) * 1e3
    res = {"workload": cfg.name, "ms_per_step": round(ms, 4), "steps": steps,
           "prefill_tflop": round(flops / 1e12, 4), "decode_gb": round(dec_bytes / 1e9, 3),
           "roofline": {"bound": "tensor+hbm", "ideal_ms": round(ideal_ms, 4), "frac": round(ideal_ms / ms, 4),
                        "peak_source": f"{c.peak_src}: {peak_t} TFLOP/s bf16, {peak_h} GB/s"},
           "gpu_launches_per_step": 3, "clocks": clk.summary()}
    if c.with_oracle:
        from oracle import attention_ref as ref
        half = args.cpu_seconds / 2
        o_chunks, l_chunks = _bf16_to_f64(oc), lsec.cpu().numpy()
        order = np.random.default_rng(17).permutation(nc)
        got_o, ref_o, got_l, ref_l, flops_done = [], [], [], [], 0.0
        t0, done = time.perf_counter(), 0
        while done < nc and (done == 0 or time.perf_counter() - t0 < half):
            b = int(order[done])
            o, lse = ref.ref_prefill_paged(d["q_chunk"][b:b + 1], [cfg.chunk_len], d["k_pool"], d["v_pool"],
                                           d["block_table"][b:b + 1], d["kv_lens"][b:b + 1], cfg.scale, True)
            ref_o.append(o[0]), ref_l.append(lse[0])
            got_o.append(o_chunks[b]), got_l.append(l_chunks[b])
            flops_done += 4.0 * cfg.head_dim * cfg.q_heads * wl.causal_pairs(cfg.chunk_len, int(d["kv_lens"][b]), True)
            done += 1
        dt = time.perf_counter() - t0
        cpu_p = _cpu_record(round(flops_done / dt / 1e12, 6), "TFLOP/s",
                            f"prefill part: {done} of {nc} chunks, all heads", dt)
        par_p = _parity(np.stack(got_o), np.stack(ref_o), np.stack(got_l), np.stack(ref_l),
                        done * cfg.q_heads * cfg.chunk_len, nc * cfg.q_heads * cfg.chunk_len, "bf16")
        dd = dict(q=d["q_dec"], k_pool=d["k_pool"], v_pool=d["v_pool"], block_table=d["block_table"][nc:],
                  kv_lens=d["kv_lens"][nc:], scale=cfg.scale)
        cpu_d, par_d = oracle_decode_sequences(dd, _bf16_to_f64(od), lsed.cpu().numpy(), half, seed=18)
        res["cpu_baseline"] = {"prefill_part": cpu_p, "decode_part": cpu_d}
        res["parity"] = {cfg.name + "_prefill": par_p, cfg.name + "_decode": par_d}
    return res


def bench_decode_steps(c: Ctx):
    """Latency of one small decode step (8 sequences of U[512, 2048] tokens,
    32/8 heads) with the host in the loop, three ways: a direct call
    (split kernel + combine launched), a replay from the CUDA graph pool, and a
    step of the persistent decode kernel. Each is timed on the host around
    call + synchronisation (or submit + wait), median over the steps."""
    import torch
    attn = c.attn
    cfg = _with_rank_seed(wl.DecodeConfig("decode_step_b8_h32kv8_d128_len512_2k", 8, 32, 8, 128, 512, 2048, 6), c.rank)
    d = wl.make_decode(cfg)
    q = _dev_bf16(d["q"])
    kc, vc = _dev_bf16(d["k_pool"]), _dev_bf16(d["v_pool"])
    bt = torch.from_numpy(d["block_table"]).cuda()
    sl = torch.from_numpy(d["kv_lens"]).cuda()
    max_len = int(d["kv_lens"].max())
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    ws = torch.empty(max(attn.decode_workspace_bytes(q, kc, vc, bt, sl, max_seq_len=max_len), 1), dtype=torch.uint8,
                     device="cuda")
    n = max(200, c.args.steps)

    def host_median(fn):
        for _ in range(20):
            fn()
        ts = []
        for _ in range(n):
            t0 = time.perf_counter()
            fn()
            ts.append((time.perf_counter() - t0) * 1e6)
        ts.sort()
        return {"median_us": round(ts[n // 2], 2), "p10_us": round(ts[n // 10], 2), "p90_us": round(ts[(9 * n) // 10], 2)}

    def direct():
        attn.decode_paged(q, kc, vc, bt, sl, cfg.scale, max_seq_len=max_len, out=out, lse=lse, workspace=ws)
        torch.cuda.synchronize()

    res = {"workload": cfg.name, "unit": "us per step (host round trip: call + synchronise)", "steps": n,
           "kv_tokens": int(d["kv_lens"].sum())}
    res["direct"] = host_median(direct)
    dev_ms = time_loop(lambda: attn.decode_paged(q, kc, vc, bt, sl, cfg.scale, max_seq_len=max_len, out=out,
                                                 lse=lse, workspace=ws), n, c.args.warmup, c.world)
    res["direct_device_back_to_back_us"] = round(dev_ms * 1e3, 2)
    pool = attn.DecodeGraphPool(q, kc, vc, bt, sl, out, lse, [1, 2, 4, 8], [512, 1024, 2048, 4096], cfg.scale)
    try:
        stream = torch.cuda.current_stream()

        def graph():
            pool.replay(cfg.batch, max_len)
            stream.synchronize()

        res["graph"] = host_median(graph)
        res["graph_bucket"] = list(pool.replay(cfg.batch, max_len))
    finally:
        pool.close()
    torch.cuda.synchronize()
    pd = attn.PersistentDecode(q, kc, vc, bt, sl, out, lse, cfg.scale)
    try:
        res["persistent"] = host_median(lambda: pd.step(cfg.batch, max_len))
    finally:
        pd.stop()
    res["gpu_launches_per_step"] = {"direct": 2, "graph": 1, "persistent": 0}
    return res


def bench_launcher_stub(c: Ctx):
    """Host-only check of the N-rank launch (no GPU work): every rank reports in."""
    t0 = time.perf_counter()
    barrier(c.world)
    dt = max_over_ranks(time.perf_counter() - t0, c.world)
    return {"metric": METRIC, "value": None, "unit": None, "n_gpus": c.world, "steps": c.args.steps,
            "warmup": c.args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "partial": "--only launcher: a host-only check of the rank launch, not a bench line"}


def run_ours(args, rank, world, local):
    from attention_tiled_exact_b200 import binding as attn
    peaks, peak_src = load_peaks()
    c = Ctx(args, rank, world, local, attn, peaks, peak_src)

    result = {}
    parity = {}
    legs = {"tiny": ("tiny", bench_tiny), "prefill16k": ("prefill_16k", bench_prefill_16k),
            "decode": ("decode", bench_decode), "decodefp8": ("decode_fp8", bench_decode_fp8),
            "mixed": ("mixed", bench_mixed), "sharedprefix": ("shared_prefix", bench_shared_prefix),
            "backward": ("backward", bench_backward), "decodesteps": ("decode_step_latency", bench_decode_steps)}
    if args.only in (None, "prefill"):
        result.update(bench_prefill(c))
        parity.update(result.pop("parity", {}))
    for key in LEGS:
        if key == "prefill" or args.only not in (None, key):
            continue
        name, fn = legs[key]
        out = fn(c)
        parity.update(out.pop("parity", {}))
        result[name] = out
    if parity:
        result["parity"] = parity
    if args.only is not None:
        result["partial"] = f"--only {args.only}: profiling run, not a bench line"
    return result


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands on the headline workload."""
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
    threads, vendor = blas_info()
    sample = (f"{heads} (batch, head) slices of {cfg.name} over {args.steps} steps "
              f"(about {per_step_budget:.1f} s each), fp64 oracle")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": cfg.name, "batch": cfg.batch, "q_heads": cfg.q_heads, "kv_heads": cfg.kv_heads,
                       "seq_len": cfg.seqlen_q, "head_dim": cfg.head_dim, "causal": cfg.causal},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "kind": "oracle", "cores": threads,
                             "blas": vendor, "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="host-time budget of the oracle sample of each workload (0: no oracle legs)")
    ap.add_argument("--only", choices=[*LEGS, "launcher"], default=None,
                    help="profiling aid: run one workload only (the line is then marked partial); "
                         "'launcher' checks the rank launch without GPU work")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="profiling aid: fewer decode sequences (default: the full 64)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus < 1:
        raise SystemExit("bench.py: --gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = dist_setup(args.gpus, need_cuda=args.only != "launcher")
    try:
        if args.only == "launcher":
            res = bench_launcher_stub(Ctx(args, rank, world, local, None, {}, "none"))
        else:
            res = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
