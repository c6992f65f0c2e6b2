#!/usr/bin/env python
"""Benchmark of the TurboQuant compressed-KV hot path on B200.

One step = the whole hot path over one batch of synthetic input:
  1. compress every cached key and value of the workload (rotation, Lloyd-Max
     codes, QJL signs, value group quantization, packing) in one call;
  2. decode one new query token per sequence against the packed cache
     (query prep, split-K attention, combine) in one call.
The default workload is the batched Llama-8B-like layer (32 sequences x 8 KV
heads x 32768 cached tokens, 32 query heads, K 3-bit / V 2-bit, bf16 inputs,
randomized Hadamard rotation): 839 MB of packed cache, large enough that the
decode kernel's HBM roofline is meaningful. `--workload qwen2.5-3b_8k_k3v2` runs
the Qwen2.5-3B-shaped cache (36 layers x 2 KV heads x 8192 tokens, 59 MB), whose
decode time is dominated by launch and ramp latency rather than bandwidth.

Prints ONE JSON line on rank 0. `value` is decode-attention throughput in GB/s
of packed K/V bytes read (summed over ranks, divided by the slowest rank's decode
time); compression throughput is reported beside it. The L2 cache is flushed
before each timed phase (a 256 MiB write, then a 256 MiB read that evicts the dirty lines),
since a small packed cache (the Qwen-shaped one is 59 MB) fits in L2.

`--impl reference` times the fp64 CPU oracle on this machine's host cores on a
bounded sample of the same workload (the slow baseline arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "decode-attention packed-KV GB/s (% of HBM peak); compress vectors/s"
FLUSH_BYTES = 256 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b_b32_32k_k3v2", choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged-cache timings")
    ap.add_argument("--no-varlen", action="store_true",
                    help="skip the decode timing of the same cache with sequences of varied lengths")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the kernel timings of the other workloads (the `configs` object)")
    ap.add_argument("--config-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--decode-kernel", default="auto", choices=["auto", "tcgen05", "mma", "cuda_core"],
                    help="decode kernel family (default: the library's choice for the shape)")
    ap.add_argument("--sweep", action="store_true",
                    help="compression sweep instead of the step: 1,048,576 bf16 keys at every head "
                         "dimension (64, 128, 256), key bit width (2, 3, 4) and rotation (Hadamard, Haar)")
    ap.add_argument("--decode-only", action="store_true",
                    help="decode a random packed cache of the workload's size (no bf16 inputs, no "
                         "compression, no e2e): a small process for profiler captures")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def source_sha(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "kv_cache_vector_05_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# Source files of each main kernel: a recorded ncu traffic figure applies while their hash is unchanged.
KERNEL_SOURCES = {
    "decode_mma_kernel": ("decode_mma.cu", "tq_device.cuh"),
    "decode_tc_kernel": ("decode_tc.cu", "tq_device.cuh", "tq_sm100.cuh"),
    "decode_kernel": ("decode.cu", "tq_device.cuh"),
    "compress_pipe_kernel": ("compress.cu", "tq_device.cuh", "tq_sm100.cuh"),
    "compress_q4_kernel": ("compress.cu", "tq_device.cuh", "tq_sm100.cuh"),
    "compress_kernel": ("compress.cu", "tq_device.cuh", "tq_sm100.cuh"),
}


def recorded_traffic(sha: str, units: int, kernel: str):
    """DRAM bytes of one launch over `units` units, from the committed ncu summary
    profiles/<kernel>_traffic.txt that gives DRAM bytes per unit for the same kernel and
    source hash (None if absent or stale)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("source_sha256_16") != sha or kv.get("kernel") != kernel:
        return None
    try:
        return float(kv["dram_bytes_per_unit"]) * units
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------- ranks

def max_over_ranks(x: float, world: int, device) -> float:
    """Slowest rank's value (all-reduce MAX over the default process group)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time
    (weak scaling: every rank processes the same units)."""
    return world * units_per_rank / slowest_seconds


# ---------------------------------------------------------------------- inputs

def host_inputs(w: W.Workload, rank: int):
    """bf16/fp32 K, V [units*tokens, d] and Q [batch, hq, d] as numpy fp32 arrays."""
    if w.name.startswith("qwen"):
        K = np.empty((w.units * w.tokens, w.d), np.float32)
        V = np.empty_like(K)
        for layer in range(w.batch):
            for h in range(w.hkv):
                u = layer * w.hkv + h
                k, v = W.qwen_layer_head_kv(layer, h, w.tokens, w.d)
                K[u * w.tokens:(u + 1) * w.tokens] = k
                V[u * w.tokens:(u + 1) * w.tokens] = v
    else:
        K = V = None  # drawn on the device
    Q = W.queries((w.batch, w.hq, w.d), seed=7 + rank, dtype=w.dtype)
    return K, V, Q


# ---------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        # TQ_CLOCKS_DIR keeps the raw samples where the caller wants them (default: a temp dir)
        out_dir = os.environ.get("TQ_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_bench_{os.getpid()}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", gpu_id], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception as e:  # pragma: no cover - no nvidia-smi
            log("clock sampler unavailable:", e)
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------- CPU oracle

def oracle_sample(w: W.Workload, budget_s: float, K=None, V=None, Q=None):
    """Time the fp64 oracle on whole (sequence, KV head) units of the workload.
    Returns dict(decode_gbs, compress_vps, units, decode_s, compress_s, cores)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = 1
    dr = W.method_draws(w.d, w.m)
    Pi = O.hadamard_rotation(dr["hadamard_signs"])
    c, t = O.device_codebook(w.d, w.lm_bits)
    S = dr["qjl_S"]
    if Q is None:
        Q = W.queries((w.batch, w.hq, w.d), seed=7, dtype=w.dtype)
    rec = w.k_record_bytes() + w.v_record_bytes()
    comp_s = dec_s = 0.0
    n_units = 0
    t_start = time.perf_counter()
    while n_units < w.units and (n_units == 0 or time.perf_counter() - t_start < budget_s):
        u = n_units
        b, kvh = divmod(u, w.hkv)
        if K is not None:
            k = K[u * w.tokens:(u + 1) * w.tokens].astype(np.float64)
            v = V[u * w.tokens:(u + 1) * w.tokens].astype(np.float64)
        else:
            k32, v32 = W.unit_keys_values(w, u)
            k, v = k32.astype(np.float64), v32.astype(np.float64)
        t0 = time.perf_counter()
        pk = O.compress_keys(k, Pi, c, t, S)
        pv = O.quantize_values(v, w.v_bits)
        t1 = time.perf_counter()
        O.decode_attention(Q[b, kvh * w.group:(kvh + 1) * w.group].astype(np.float64), pk, pv, Pi, c, S,
                           w.d, w.v_bits)
        t2 = time.perf_counter()
        comp_s += t1 - t0
        dec_s += t2 - t1
        n_units += 1
    return {"decode_gbs": n_units * w.tokens * rec / dec_s / 1e9,
            "compress_vps": 2 * n_units * w.tokens / comp_s,
            "units": n_units, "decode_s": dec_s, "compress_s": comp_s, "cores": cores}


def run_reference(args, w: W.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    K, V, Q = host_inputs(w, 0)
    per_step = max(args.cpu_seconds / max(args.steps, 1), 0.05)
    for _ in range(args.warmup):
        oracle_sample(w, 0.0, K, V, Q)
    res = [oracle_sample(w, per_step, K, V, Q) for _ in range(args.steps)]
    dec_s = sum(r["decode_s"] for r in res)
    comp_s = sum(r["compress_s"] for r in res)
    units = sum(r["units"] for r in res)
    rec = w.k_record_bytes() + w.v_record_bytes()
    gbs = units * w.tokens * rec / dec_s / 1e9
    sample = (f"{units} (sequence, KV head) units over {args.steps} steps; each: compress "
              f"{w.tokens} keys + {w.tokens} values, decode {w.group} query heads (fp64 numpy oracle)")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * (dec_s + comp_s) / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "kv_heads": w.hkv, "q_heads": w.hq,
                   "tokens": w.tokens, "head_dim": w.d, "k_bits": w.k_bits, "v_bits": w.v_bits,
                   "rotation": w.rotation, "packed_bytes": w.packed_bytes(),
                   "l2": "flushed before each timed phase: 256 MiB write, then 256 MiB read",
                   "parallelism": f"dp{args.gpus} (independent replicas)"},
        "compress": {"value": 2 * units * w.tokens / comp_s, "unit": "vectors/s"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": res[0]["cores"], "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU arm

SIDE_WORKLOADS = ("single_head_d128_n4096", "qwen2.5-3b_8k_k3v2", "long_1m_k4v4")
KERNEL_IDS = {"auto": 0, "tcgen05": 1, "mma": 2, "cuda_core": 3}
KERNEL_NAMES = {1: "tcgen05", 2: "mma", 3: "cuda_core"}
# main attention kernel of each decode family (the one the library brackets with profile events)
DECODE_KERNEL_OF = {1: "decode_tc_kernel", 2: "decode_mma_kernel", 3: "decode_kernel"}


def time_side_workload(T, torch, w: W.Workload, steps: int, warmup: int, dev, flush_l2, peak: float):
    """Kernel times of one compression call and one decode call of workload `w` (inputs
    drawn by its recipe; L2 flushed before every timed launch; CUDA events around the main
    kernel of each call, recorded by the library on the launching stream)."""
    dr = W.method_draws(w.d, w.m)
    c, t = T.tq_lloyd_max_codebook(w.d, w.lm_bits)
    ctx = T.tq_codebook_load(w.d, w.lm_bits, w.v_bits, c, t, dr["qjl_S"], hadamard_signs=dr["hadamard_signs"])
    n_vec = w.units * w.tokens
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if w.name.startswith("single_head"):
        Kh, Vh, Qh = W.single_head_kvq(w.tokens, w.d, w.hq)
        K, V = torch.from_numpy(Kh).to(dev).to(tdt), torch.from_numpy(Vh).to(dev).to(tdt)
        Q = torch.from_numpy(Qh).to(dev).to(tdt).view(w.batch, w.hq, w.d)
    else:
        if w.name.startswith("qwen"):
            Kh, Vh, _ = host_inputs(w, 0)
            K, V = torch.from_numpy(Kh).to(dev).to(tdt), torch.from_numpy(Vh).to(dev).to(tdt)
            del Kh, Vh
        else:
            K = W.device_normal((n_vec, w.d), seed=3000, device=dev).to(tdt)
            V = W.device_normal((n_vec, w.d), seed=4000, device=dev).to(tdt)
        Q = torch.from_numpy(W.queries((w.batch, w.hq, w.d), seed=7, dtype=w.dtype)).to(dev).to(tdt)
    packed = T.tq_compress_kv(ctx, K, V)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=dev)
    ws = torch.empty(T.tq_decode_workspace_bytes(ctx, w.batch, w.hq, w.hkv, w.tokens), dtype=torch.uint8,
                     device=dev)
    E = torch.cuda.Event
    comp, dec = [], []
    for it in range(warmup + steps):
        e = [E(enable_timing=True) for _ in range(4)]
        for ev in e:
            ev.record()
        flush_l2()
        T.tq_set_profile_events(ctx, e[0], e[1])
        T.tq_compress_kv(ctx, K, V, **packed)
        flush_l2()
        T.tq_set_profile_events(ctx, e[2], e[3])
        T.tq_decode_attention(ctx, Q, packed, w.batch, w.hq, w.hkv, w.tokens, out=out, workspace=ws)
        T.tq_set_profile_events(ctx, None, None)
        if it >= warmup:
            comp.append(e)
    torch.cuda.synchronize()
    T.tq_check_device(ctx)
    ck = statistics.median(e[0].elapsed_time(e[1]) for e in comp) / 1e3
    dk = statistics.median(e[2].elapsed_time(e[3]) for e in comp) / 1e3
    packed_bytes = w.packed_bytes()
    comp_bytes = 2 * n_vec * w.d * (2 if w.dtype == "bf16" else 4) + packed_bytes
    fam = T.tq_decode_kernel_for(ctx, w.hq, w.hkv)
    ctx.close()
    return {"decode_kernel": DECODE_KERNEL_OF.get(fam), "batch": w.batch, "kv_heads": w.hkv, "q_heads": w.hq, "tokens": w.tokens, "k_bits": w.k_bits,
            "v_bits": w.v_bits, "dtype": w.dtype, "packed_bytes": packed_bytes, "steps": steps,
            "compress_kernel_us": ck * 1e6, "compress_vectors_per_s": 2 * n_vec / ck,
            "compress_gbs": comp_bytes / ck / 1e9, "compress_frac": comp_bytes / ck / 1e9 / peak,
            "decode_kernel_us": dk * 1e6, "decode_gbs": packed_bytes / dk / 1e9,
            "decode_frac": packed_bytes / dk / 1e9 / peak,
            "timing": "median over steps of CUDA events around each call's main kernel, L2 flushed before each"}


def run_ours(args, w: W.Workload):
    import torch
    import torch.distributed as dist
    import kv_cache_vector_05_b200 as T

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def slowest(x: float) -> float:
        return max_over_ranks(x, world, dev)

    # --- method tables and inputs
    dr = W.method_draws(w.d, w.m)
    c, t = T.tq_lloyd_max_codebook(w.d, w.lm_bits)
    ctx = T.tq_codebook_load(w.d, w.lm_bits, w.v_bits, c, t, dr["qjl_S"], hadamard_signs=dr["hadamard_signs"])
    T.tq_set_decode_kernel(ctx, KERNEL_IDS[args.decode_kernel])
    fam = T.tq_decode_kernel_for(ctx, w.hq, w.hkv)
    if fam < 0:
        raise SystemExit(f"the {args.decode_kernel} decode kernel does not take workload {w.name}")
    n_vec = w.units * w.tokens
    if args.decode_only:
        args.no_e2e = args.no_cpu_baseline = True
    Kh, Vh, Qh = host_inputs(w, rank) if not args.decode_only else (None, None, W.queries(
        (w.batch, w.hq, w.d), seed=7 + rank, dtype=w.dtype))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if args.decode_only:
        K = V = None
    elif Kh is not None:
        K = torch.from_numpy(Kh).to(dev).to(tdt)
        V = torch.from_numpy(Vh).to(dev).to(tdt)
        del Kh, Vh
    else:
        K = W.device_normal((n_vec, w.d), seed=1000 + rank, device=dev).to(tdt)
        V = W.device_normal((n_vec, w.d), seed=2000 + rank, device=dev).to(tdt)
    Q = torch.from_numpy(Qh).to(dev).to(tdt)
    if args.decode_only:
        pk = W.random_packed_cache(n_vec, w.d, w.lm_bits, w.m, w.v_bits, seed=11 + rank)
        packed = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                                      else np.ascontiguousarray(v)).to(dev) for k, v in pk.items()}
        del pk
    else:
        packed = None
    packed = packed or {
        "k_codes": torch.empty((n_vec, w.lm_bits * w.d // 8), dtype=torch.uint8, device=dev),
        "k_signs": torch.empty((n_vec, w.m // 8), dtype=torch.uint8, device=dev),
        "k_norms": torch.empty((n_vec, 2), dtype=torch.int16, device=dev),
        "v_codes": torch.empty((n_vec, w.v_bits * w.d // 8), dtype=torch.uint8, device=dev),
        "v_params": torch.empty((n_vec, w.d // 32, 2), dtype=torch.int16, device=dev),
    }
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=dev)
    ws = torch.empty(T.tq_decode_workspace_bytes(ctx, w.batch, w.hq, w.hkv, w.tokens), dtype=torch.uint8,
                     device=dev)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_src = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # Write a buffer larger than L2, then read another one: the read evicts the
        # dirty lines the write left behind, so the next timed kernel starts with a
        # cold L2 and no write-back traffic of the flush in its own time.
        flush_buf.zero_()
        flush_src.sum()
    packed_bytes = n_vec * (w.k_record_bytes() + w.v_record_bytes())
    in_bytes = 2 * n_vec * w.d * (2 if w.dtype == "bf16" else 4)

    def compress():
        if not args.decode_only:
            T.tq_compress_kv(ctx, K, V, **packed)

    def decode():
        T.tq_decode_attention(ctx, Q, packed, w.batch, w.hq, w.hkv, w.tokens, out=out, workspace=ws)

    E = torch.cuda.Event

    def run_steps(n, kernel_events):
        """n steps; with kernel_events the library also brackets its main kernels
        (this separates the decode kernel from its prep launch, so those steps time
        the kernels alone and are kept out of the call timings)."""
        evs = []
        for _ in range(n):
            e = [E(enable_timing=True) for _ in range(8)]
            for ev in (e[1], e[2], e[5], e[6]):
                ev.record()  # torch creates the CUDA event lazily; the library re-records it
            flush_l2()
            e[0].record()
            if kernel_events:
                T.tq_set_profile_events(ctx, e[1], e[2])
            compress()
            e[3].record()
            flush_l2()
            e[4].record()
            if kernel_events:
                T.tq_set_profile_events(ctx, e[5], e[6])
            decode()
            e[7].record()
            if kernel_events:
                T.tq_set_profile_events(ctx, None, None)
            evs.append(e)
        return evs

    run_steps(args.warmup, True)
    run_steps(args.warmup, False)
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_id = vis.split(",")[local] if vis else str(local)
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    time.sleep(1.0)
    run_steps(max(3, args.warmup // 2), False)

    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    evs = run_steps(args.steps, False)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    # the same number of steps again, with the main kernels bracketed by events
    kevs = run_steps(args.steps, True)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None

    comp = [e[0].elapsed_time(e[3]) for e in evs]
    comp_k = [e[1].elapsed_time(e[2]) for e in kevs]
    dec = [e[4].elapsed_time(e[7]) for e in evs]
    dec_k = [e[5].elapsed_time(e[6]) for e in kevs]
    dec_total = slowest(sum(dec) / 1e3)
    comp_total = slowest(sum(comp) / 1e3)
    dec_k_mean = slowest(statistics.fmean(dec_k) / 1e3)
    gbs = job_throughput(packed_bytes * args.steps, world, dec_total) / 1e9
    vps = job_throughput(2 * n_vec * args.steps, world, comp_total) if not args.decode_only else None

    # --- the same cache through the append / paged calls: the packed arrays scattered over
    # pages of 512 tokens in a shuffled order (block table); compression through the
    # matching slot map. Kernel times, L2 flushed before each, like the main loop.
    paged_line = None
    if not args.no_paged:
        P = 512
        mp = (w.tokens + P - 1) // P
        n_pages = w.units * mp
        gen = torch.Generator(device=dev)
        gen.manual_seed(5 + rank)
        table = torch.randperm(n_pages, generator=gen, device=dev).view(w.units, mp).to(torch.int32)
        tok = torch.arange(w.tokens, device=dev)
        rows = (table[:, tok // P].long() * P + tok % P).reshape(-1)   # record row of token (u, t)
        paged = {k: torch.empty((n_pages * P,) + tuple(v.shape[1:]), dtype=v.dtype, device=dev)
                 for k, v in packed.items()}
        for k in packed:
            paged[k].index_copy_(0, rows, packed[k])
        bt = table.view(w.batch, w.hkv, mp).contiguous()
        pdec, pcomp = [], []
        for it in range(args.warmup + args.steps):
            e = [E(enable_timing=True) for _ in range(4)]
            for ev in e:
                ev.record()
            flush_l2()
            T.tq_set_profile_events(ctx, e[0], e[1])
            T.tq_decode_attention_paged(ctx, Q, paged, w.batch, w.hq, w.hkv, w.tokens, bt, P, n_pages,
                                        out=out, workspace=ws)
            if not args.decode_only:
                flush_l2()
                T.tq_set_profile_events(ctx, e[2], e[3])
                T.tq_compress_kv_slots(ctx, K, V, rows, paged)
            T.tq_set_profile_events(ctx, None, None)
            if it >= args.warmup:
                pdec.append(e)
        torch.cuda.synchronize()
        T.tq_check_device(ctx)
        pd = slowest(statistics.fmean(e[0].elapsed_time(e[1]) for e in pdec) / 1e3)
        paged_line = {"page_size": P, "pages": n_pages, "block_order": "shuffled",
                      "decode_main_kernel_ms": pd * 1e3,
                      "decode_gbs": job_throughput(packed_bytes, world, pd) / 1e9}
        if not args.decode_only:
            pc = slowest(statistics.fmean(e[2].elapsed_time(e[3]) for e in pdec) / 1e3)
            paged_line.update({"compress_slots_kernel_ms": pc * 1e3,
                               "compress_slots_vectors_per_s": job_throughput(2 * n_vec, world, pc)})
        del paged, rows, table, bt

    # --- the same cache, each sequence holding a seeded uniform number of tokens in
    # [tokens / 2, tokens] (seq_lens): decode kernel time and GB/s of the tokens present.
    varlen_line = None
    if not args.no_varlen:
        lens = np.random.default_rng(21 + rank).integers(w.tokens // 2, w.tokens + 1, w.batch)
        lens_t = torch.from_numpy(lens.astype(np.int32)).to(dev)
        vdec = []
        for it in range(args.warmup + args.steps):
            e = [E(enable_timing=True) for _ in range(2)]
            for ev in e:
                ev.record()
            flush_l2()
            T.tq_set_profile_events(ctx, e[0], e[1])
            T.tq_decode_attention(ctx, Q, packed, w.batch, w.hq, w.hkv, w.tokens, seq_lens=lens_t, out=out,
                                  workspace=ws)
            T.tq_set_profile_events(ctx, None, None)
            if it >= args.warmup:
                vdec.append(e)
        torch.cuda.synchronize()
        T.tq_check_device(ctx)
        vd = slowest(statistics.fmean(e[0].elapsed_time(e[1]) for e in vdec) / 1e3)
        present = int(lens.sum()) * w.hkv * (w.k_record_bytes() + w.v_record_bytes())
        varlen_line = {"lengths": "uniform in [tokens / 2, tokens] per sequence (seeded)",
                       "tokens_present_fraction": float(lens.sum()) / (w.batch * w.tokens),
                       "decode_main_kernel_ms": vd * 1e3,
                       "decode_gbs": job_throughput(present, world, vd) / 1e9}

    # --- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        Kp = K.cpu().pin_memory()
        Vp = V.cpu().pin_memory()
        Qp = Q.cpu().pin_memory()
        outp = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        Kd, Vd, Qd = torch.empty_like(K), torch.empty_like(V), torch.empty_like(Q)

        def e2e_step():
            Kd.copy_(Kp, non_blocking=True)
            Vd.copy_(Vp, non_blocking=True)
            Qd.copy_(Qp, non_blocking=True)
            T.tq_compress_kv(ctx, Kd, Vd, **packed)
            T.tq_decode_attention(ctx, Qd, packed, w.batch, w.hq, w.hkv, w.tokens, out=out, workspace=ws)
            outp.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        s0, s1 = E(enable_timing=True), E(enable_timing=True)
        s0.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e2e_s = slowest(s0.elapsed_time(s1) / 1e3)
        h2d = Kp.numel() * Kp.element_size() + Vp.numel() * Vp.element_size() + Qp.numel() * Qp.element_size()
        e2e = {"value": job_throughput(packed_bytes * args.e2e_steps, world, e2e_s) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(outp.numel() * 4),
               "ms_per_step": 1e3 * e2e_s / args.e2e_steps}

    # our kernels per step: compress (1) + decode (query prep + attention + combine)
    launches_per_step = (0 if args.decode_only else 1) + 3

    # The other tensor-core decode family on the same cache, when it takes the shape: its
    # main kernel alone, L2 flushed before each launch (reported beside the chosen one).
    alt = {}
    if rank == 0 and world == 1 and not args.no_configs:
        for f2 in (1, 2):
            if f2 == fam:
                continue
            T.tq_set_decode_kernel(ctx, f2)
            if T.tq_decode_kernel_for(ctx, w.hq, w.hkv) != f2:
                continue
            ws2 = torch.empty(T.tq_decode_workspace_bytes(ctx, w.batch, w.hq, w.hkv, w.tokens), dtype=torch.uint8,
                              device=dev)
            ts = []
            for it in range(3 + args.config_steps):
                e = [E(enable_timing=True) for _ in range(2)]
                for ev in e:
                    ev.record()
                flush_l2()
                T.tq_set_profile_events(ctx, e[0], e[1])
                T.tq_decode_attention(ctx, Q, packed, w.batch, w.hq, w.hkv, w.tokens, out=out, workspace=ws2)
                T.tq_set_profile_events(ctx, None, None)
                if it >= 3:
                    ts.append(e)
            torch.cuda.synchronize()
            T.tq_check_device(ctx)
            k_s = statistics.median(e[0].elapsed_time(e[1]) for e in ts) / 1e3
            alt[KERNEL_NAMES[f2]] = {"kernel": DECODE_KERNEL_OF[f2], "kernel_us": k_s * 1e6,
                                     "gbs": packed_bytes / k_s / 1e9, "steps": args.config_steps}
            del ws2
        T.tq_set_decode_kernel(ctx, KERNEL_IDS[args.decode_kernel])

    side = None
    if rank == 0 and world == 1 and not args.no_configs and not args.decode_only:
        peak, _ = measured_peaks()
        side = {}
        for name in SIDE_WORKLOADS:
            if name == w.name:
                continue
            side[name] = time_side_workload(T, torch, W.WORKLOADS[name], args.config_steps, 3, dev, flush_l2, peak)
            log(f"config {name}: compress {side[name]['compress_kernel_us']:.1f} us, "
                f"decode {side[name]['decode_kernel_us']:.1f} us ({side[name]['decode_gbs']:.0f} GB/s)")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Kh2, Vh2, _ = host_inputs(w, 0) if w.name.startswith("qwen") else (None, None, None)
        r = oracle_sample(w, args.cpu_seconds, Kh2, Vh2, Qh)
        cpu = {"value": r["decode_gbs"], "unit": "GB/s", "cores": r["cores"], "kind": "oracle",
               "sample": (f"{r['units']} of {w.units} (sequence, KV head) units: compress {w.tokens} keys + "
                          f"{w.tokens} values and decode {w.group} query heads each; fp64 numpy oracle; "
                          f"compress {r['compress_vps']:.4g} vectors/s")}

    if rank == 0:
        peak, peak_kind = measured_peaks()
        units_dec = w.units * w.tokens  # (token, KV head) pairs
        dkern = DECODE_KERNEL_OF[fam]
        dsha = source_sha(KERNEL_SOURCES[dkern])
        roof_dec = {"kernel": dkern, "bound": "hbm", "achieved": packed_bytes / dec_k_mean / 1e9,
                    "peak": peak, "unit": "GB/s", "frac": packed_bytes / dec_k_mean / 1e9 / peak,
                    "peak_kind": peak_kind, "alg_bytes_per_launch": packed_bytes,
                    "alg_bytes_per_unit": w.k_record_bytes() + w.v_record_bytes(), "unit_of_work": "token x KV head",
                    "traffic": recorded_traffic(dsha, units_dec, dkern),
                    "source_sha256_16": dsha}
        roof = roof_dec
        if not args.decode_only:
            # The compression kernel takes most of a step, so it is the step's dominant kernel.
            comp_bytes = in_bytes + packed_bytes
            comp_k_mean = statistics.fmean(comp_k) / 1e3
            # d = m = 128 with the Hadamard rotation: bf16 keys (symmetric Lloyd-Max codebook) take
            # the pipelined tensor-core kernel, fp32 keys the four-lanes-per-vector one
            tc = w.d == 128 and w.m == 128 and w.rotation == "hadamard"
            ckern = ("compress_pipe_kernel" if w.dtype == "bf16" else "compress_q4_kernel") if tc \
                else "compress_kernel"
            csha = source_sha(KERNEL_SOURCES[ckern])
            roof = {"kernel": ckern, "bound": "hbm", "achieved": comp_bytes / comp_k_mean / 1e9, "peak": peak,
                    "unit": "GB/s", "frac": comp_bytes / comp_k_mean / 1e9 / peak, "peak_kind": peak_kind,
                    "alg_bytes_per_launch": comp_bytes, "alg_bytes_per_unit": comp_bytes // n_vec,
                    "unit_of_work": "key + value vector pair",
                    "traffic": recorded_traffic(csha, n_vec, ckern),
                    "source_sha256_16": csha}
        line = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * (dec_total + comp_total) / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "kv_heads": w.hkv, "q_heads": w.hq,
                       "tokens": w.tokens, "head_dim": w.d, "k_bits": w.k_bits, "v_bits": w.v_bits,
                       "rotation": w.rotation, "packed_bytes": packed_bytes,
                       "l2": "flushed before each timed phase: 256 MiB write, then 256 MiB read",
                       "parallelism": f"dp{world} (independent replicas)"},
            "pct_of_hbm_peak": 100.0 * gbs / peak,
            "compress": None if args.decode_only else {
                "value": vps, "unit": "vectors/s (keys + values)",
                "gbs": world * (in_bytes + packed_bytes) * args.steps / comp_total / 1e9,
                "kernel_ms": statistics.fmean(comp_k)},
            "decode_ms": {"call": dec_total * 1e3 / args.steps, "main_kernel": dec_k_mean * 1e3,
                          "main_kernel_timing": "separate loop of `steps` steps with events around the kernel"},
            "paged": paged_line,
            "varlen": varlen_line,
            "roofline": roof,
            "roofline_decode": roof_dec,
            "decode_kernel": KERNEL_NAMES[fam],
            "decode_alternatives": alt or None,
            "configs": side,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "wall_s": wall,
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


def run_sweep(args):
    """Keys-only compression of W.SWEEP_VECTORS bf16 N(0,1) keys for every (d, b, rotation)
    (b total key bits: b - 1 Lloyd-Max bits + 1 QJL bit, m = d). Each configuration is
    timed over `steps` launches with CUDA events, the L2 flushed before each; one JSON line
    with a row per configuration (median launch time, keys/s, GB/s of algorithmic bytes:
    2d bytes of bf16 in, the packed record out)."""
    import torch
    import kv_cache_vector_05_b200 as T
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = measured_peaks()
    n = W.SWEEP_VECTORS
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_src = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    rows = []
    for d in W.SWEEP_D:
        K = W.device_normal((n, d), seed=1, device=dev).to(torch.bfloat16)
        dr = W.method_draws(d, d)
        for b in W.SWEEP_BITS:
            lm = b - 1
            c, t = T.tq_lloyd_max_codebook(d, lm)
            for rot in ("hadamard", "haar"):
                haar = T.tq_haar_from_gaussian(dr["haar_gaussian"]) if rot == "haar" else None
                ctx = T.tq_codebook_load(d, lm, 2, c, t, dr["qjl_S"], rotation=rot,
                                         hadamard_signs=dr["hadamard_signs"], haar=haar)
                out = T.tq_compress_kv(ctx, K, None)
                for _ in range(max(3, args.warmup)):
                    T.tq_compress_kv(ctx, K, None, **out)
                ms = []
                for _ in range(args.steps):
                    flush_buf.zero_()
                    flush_src.sum()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    T.tq_compress_kv(ctx, K, None, **out)
                    e1.record()
                    torch.cuda.synchronize()
                    ms.append(e0.elapsed_time(e1))
                T.tq_check_device(ctx)
                med = statistics.median(ms)
                rec = lm * d // 8 + d // 8 + 4
                alg = n * (2 * d + rec)
                rows.append({"d": d, "b": b, "rotation": rot, "ms": med, "keys_per_s": n / (med * 1e-3),
                             "gbs": alg / (med * 1e-3) / 1e9, "frac": alg / (med * 1e-3) / 1e9 / peak,
                             "alg_bytes_per_key": 2 * d + rec})
                log(f"sweep d={d} b={b} {rot}: {med:.4f} ms, {rows[-1]['gbs']:.0f} GB/s")
                ctx.close()
        del K
    print(json.dumps({"metric": "compress keys/s (sweep)", "unit": "keys/s", "vectors": n, "dtype": "bf16",
                      "steps": args.steps, "warmup": max(3, args.warmup), "peak_gbs": peak, "peak_kind": peak_kind,
                      "l2": "flushed before each launch: 256 MiB write, then 256 MiB read", "sweep": rows}))


def main():
    args = parse()
    w = W.WORKLOADS[args.workload]
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
