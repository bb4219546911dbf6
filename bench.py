#!/usr/bin/env python
"""Benchmark of the compressed-KV decode hot path on B200.

A step is one decode step of one attention layer of the workload: the new token's K and V
are quantised into the packed cache (tq_quantize_kv at position T-1), then decode attention
runs over all T cached tokens (tq_decode_attention: split-K kernel + combine). The headline
value is packed-KV bytes read per step / step time (GB/s), summed over ranks (one replica
per GPU, weak scaling). Inputs are seeded synthetic tensors resident in HBM; the packed
cache (419 MB for the default workload) is larger than the 126 MB L2, so no flush is needed.

Side measurements on rank 0 (outside the timed loop): the decode call alone (roofline), the
bulk quantise of the whole layer (Mtok/s), the bf16 kernel of the same design (speedup),
an end-to-end run from pinned host buffers, the oracle on a bounded sample (cpu_baseline),
and nvidia-smi clocks sampled during the timed loop.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import csv
import dataclasses
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn GB/s & % of B200 HBM peak on packed KV; quantize Mtok/s"
DEFAULT_WORKLOAD = "llama3_8b_decode_32k"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-side", action="store_true", help="skip side measurements")
    ap.add_argument("--T", type=int, default=0,
                    help="override the context length (profiling runs on smaller cases)")
    ap.add_argument("--paged-case", type=int, default=0,
                    help="T: run the Llama-3.1-8B-shaped decode (batch 16, K4/V2) over a T-position paged "
                         "cache (64-position pages, seeded scatter) twice and exit (profiling)")
    ap.add_argument("--prefill-case", default="",
                    help="T,Lq[,e2m1]: run one prefill chunk of Lq queries at the end of a T-position cache "
                         "(Llama-3.1-8B shape, batch 4, 4-bit keys (Lloyd-Max, or E2M1 with ',e2m1'), "
                         "2-bit values) and exit (profiling)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def kernel_traffic():
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary, if the
    decode source is unchanged since the capture (else null)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("sources_sha256") != decode_sources_digest():
        return None
    return rec.get("dram_bytes_per_launch")


def _code_only(src: str) -> str:
    """C++ source without comments and whitespace (string literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            if not src[i].isspace():
                out.append(src[i])
            i += 1
    return "".join(out)


DECODE_SOURCES = ("decode_mma.cu", "decode_mse_common.cuh", "mma_ops.cuh", "tq_device.cuh")


def decode_sources_digest() -> str:
    """sha256 over the code (comments and whitespace removed) of the bench's dominant kernel's
    sources (the tensor-core decode)."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "quantized_decode_attention_kv_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


ARITH_MSE = ("u8 packed codes; scores on int8 tensor cores (16-bit fixed-point centroids x 24-bit "
             "fixed-point queries, int32 accumulation), P.V on f16 tensor cores with f32 "
             "accumulation; f32 softmax")
ARITH_PROD = ("u8 packed codes and sign bits as exact +-1 f16 operands; scores and P.V on f16 tensor "
              "cores with f32 accumulation (hi/lo split query side); f32 softmax")


class Clocks:
    """nvidia-smi samples every 100 ms while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        load = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ oracle (CPU) arm
def oracle_sample(w, heads: int):
    """Records and queries for `heads` (b, KV-head) slices of the workload, full context."""
    import numpy as np

    import oracle as O
    from quantized_decode_attention_kv_b200.workloads import make_inputs
    K, V, q = make_inputs(w, B=1, Hkv=heads, Hq=heads * w.G)
    samples = []
    for h in range(heads):
        Kn = K[0, h].float().numpy().astype(np.float64)
        Vn = V[0, h].float().numpy().astype(np.float64)
        kr = O.quantize(Kn, w.k_bits, w.k_mode, seed=w.seed, qjl_seed=w.qjl_seed, m=w.qjl_m or None)
        vr = O.quantize(Vn, w.v_bits, w.v_mode, seed=w.seed, qjl_seed=w.qjl_seed, m=w.qjl_m or None)
        qs = q[:, h * w.G:(h + 1) * w.G].float().numpy().astype(np.float64)
        samples.append((qs, kr, vr))
    rec_bytes = (O.record_bytes(w.d, w.k_bits, w.k_mode, w.qjl_m or None)
                 + O.record_bytes(w.d, w.v_bits, w.v_mode, w.qjl_m or None))
    return samples, rec_bytes * w.T


def oracle_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:  # noqa: BLE001
        blas = 1
    return blas, len(os.sched_getaffinity(0))


def time_oracle_decode(w, budget_s: float = 12.0):
    import oracle as O
    samples, per_head_bytes = oracle_sample(w, heads=2)
    reps, t0 = 0, time.perf_counter()
    while True:
        qs, kr, vr = samples[reps % len(samples)]
        O.decode_compressed(qs, [kr], [vr], 1, 1, w.scale)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 200:
            break
    blas, aff = oracle_cores()
    return {"value": per_head_bytes * reps / el / 1e9, "unit": "GB/s", "cores": blas,
            "kind": "oracle",
            "sample": (f"{reps} oracle decode steps of one (batch, KV head) slice each: dequantise "
                       f"{w.T} K and V records (float64, explicit Hadamard) + two-pass softmax for "
                       f"{w.G} query heads; {per_head_bytes} packed bytes per slice; "
                       f"{blas} BLAS threads of {aff} cores in affinity")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS
    import oracle as O
    w = WORKLOADS[args.workload]
    samples, per_head_bytes = oracle_sample(w, heads=2)
    times = []
    for i in range(args.warmup + args.steps):
        qs, kr, vr = samples[i % len(samples)]
        t0 = time.perf_counter()
        O.decode_compressed(qs, [kr], [vr], 1, 1, w.scale)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    step = statistics.mean(times)
    value = per_head_bytes / step / 1e9
    blas, aff = oracle_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "sample": "one (batch, KV head) slice per step, full context",
                       "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "k_bits": w.k_bits,
                       "v_bits": w.v_bits},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": blas, "kind": "oracle",
                             "sample": f"oracle decode of one (b, KV head) slice of {w.T} tokens per step; "
                                       f"{blas} BLAS threads of {aff} cores"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ CUDA arm
def run_ours(args):
    import torch

    from quantized_decode_attention_kv_b200 import replicas as R
    from quantized_decode_attention_kv_b200 import tq
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs

    rank, local, world = R.env_ranks()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    R.init("nccl", world, torch.device("cuda", local))

    def barrier():
        R.barrier(world)

    w = WORKLOADS[args.workload]
    if args.T:
        w = dataclasses.replace(w, T=args.T)
    K, V, q = make_inputs(w, device="cuda", layer=R.replica_layer(rank))
    cache = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, w.k_mode, w.v_mode, w.qjl_m,
                       w.qjl_m, seed=w.seed, qjl_seed=w.qjl_seed)
    tq.tq_quantize_kv(K, V, cache)  # prefill the whole context
    k_new = K[:, :, w.T - 1:].contiguous()
    v_new = V[:, :, w.T - 1:].contiguous()
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, w.Hq, w.T))
    stream = torch.cuda.current_stream()
    packed = cache.packed_bytes(w.T)

    def step():
        tq.tq_quantize_kv(k_new, v_new, cache, t_offset=w.T - 1, stream=stream)
        tq.tq_decode_attention(q, cache, w.T, w.scale, out, ws, stream=stream)

    clocks = Clocks(local)
    with clocks:
        # the W warm-up steps run inside the clock-sampling window, continued until the GPU has
        # been busy for SETTLE_S (the sampler's start-up leaves it idle, and the first steps
        # after an idle spell run at lower clocks)
        warm = 0
        t_warm = time.perf_counter()
        while warm < args.warmup or time.perf_counter() - t_warm < SETTLE_S:
            for _ in range(10):
                step()
            warm += 10
            torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = R.max_over_ranks(e0.elapsed_time(e1) / args.steps, world, device="cuda")
    value = R.job_throughput(packed, world, ms * 1e-3) / 1e9
    nq, nd = tq.tq_launch_counts(cache, k_new.dtype, 1, w.Hq, w.T)
    launches_per_step = nq + nd

    side = {}
    if rank == 0 and not args.no_side:
        side = side_measurements(args, w, tq, torch, K, V, q, cache, out, ws, k_new, v_new, packed, stream)
    barrier()
    R.finish(world)
    if rank != 0:
        return
    hbm, hbm_src = peaks()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "warmup_steps_run": warm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8+f16-mma/f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T,
                   "k": f"{w.k_bits}-bit {'MSE' if w.k_mode == 0 else 'PROD'}",
                   "v": f"{w.v_bits}-bit {'MSE' if w.v_mode == 0 else 'PROD'}",
                   "packed_bytes_per_step": packed,
                   "step": "quantise 1 new token (K,V) + decode attention over T tokens",
                   "arithmetic": ARITH_MSE if w.k_mode == 0 else ARITH_PROD,
                   "l2": "no flush: packed cache per step larger than the 126 MB L2",
                   "parallelism": f"{world} independent replica(s), one per GPU"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if side:
        dec_gbs = packed / side["decode_s"] / 1e9
        line["roofline"] = {"bound": "hbm", "achieved": dec_gbs, "peak": hbm, "unit": "GB/s",
                            "frac": dec_gbs / hbm, "traffic": kernel_traffic(),
                            "kernel": "tq_decode_attention (split-K kernel + combine), CUDA events",
                            "peak_source": hbm_src}
        line["e2e"] = side["e2e"]
        line["cpu_baseline"] = side["cpu_baseline"]
        line["decode_us"] = side["decode_s"] * 1e6
        line["quantize"] = side["quantize"]
        line["bf16_decode"] = side["bf16"]
        line["speedup_vs_bf16"] = side["bf16"]["us"] / (side["decode_s"] * 1e6)
        if "ragged" in side:
            line["ragged_decode"] = side["ragged"]
        if "paged" in side:
            line["paged_decode"] = side["paged"]
        if "k4v3" in side:
            line["decode_3p5bit"] = side["k4v3"]
        if "boundary_flips" in side:
            line["boundary_flips"] = side["boundary_flips"]
        line["configs"] = side.get("configs", {})
        line["prefill"] = side.get("prefill", {})
    print(json.dumps(line), flush=True)


MIN_CALLS, MIN_SECONDS = 200, 0.5
SETTLE_S = 0.05  # device-busy time of the warm-up before the timed steps


def _time(fn, stream, torch, min_calls=MIN_CALLS, min_s=MIN_SECONDS):
    """Mean device time of one call of fn (CUDA events on the launching stream) over at least
    min_calls calls and at least min_s seconds, after three warm-up calls."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(3):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    est = max(e0.elapsed_time(e1) / 3 * 1e-3, 1e-7)
    reps = max(min_calls, int(min_s / est) + 1)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps * 1e-3


def side_measurements(args, w, tq, torch, K, V, q, cache, out, ws, k_new, v_new, packed, stream):
    hbm, _ = peaks()
    res = {}
    # decode call alone (split-K kernel + combine)
    res["decode_s"] = _time(lambda: tq.tq_decode_attention(q, cache, w.T, w.scale, out, ws, stream=stream),
                            stream, torch)
    # bulk quantise of the whole layer: B*T token positions, all KV heads, K and V
    qclk = Clocks(torch.cuda.current_device())
    with qclk:
        qs = _time(lambda: tq.tq_quantize_kv(K, V, cache, stream=stream), stream, torch, min_calls=20)
    in_bytes = (K.numel() + V.numel()) * K.element_size()
    q_bytes = in_bytes + packed
    res["quantize"] = {"us": qs * 1e6, "mtok_s": w.B * w.T / qs / 1e6, "gbs": q_bytes / qs / 1e9,
                       "frac": q_bytes / qs / 1e9 / hbm, "bytes": q_bytes,
                       "token": "one (sequence, position) of one layer: all KV heads, K and V",
                       "clocks": qclk.summary()}
    # the same split-K design over the unquantised bf16 cache
    if K.dtype == torch.bfloat16:
        wsb = tq.workspace(tq.tq_decode_bf16_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.d))
        qb = q.to(torch.bfloat16)
        bs = _time(lambda: tq.tq_decode_attention_bf16(qb, K, V, w.T, w.scale, out, wsb, stream=stream),
                   stream, torch)
        bbytes = (K.numel() + V.numel()) * 2
        res["bf16"] = {"us": bs * 1e6, "gbs": bbytes / bs / 1e9, "frac": bbytes / bs / 1e9 / hbm,
                       "bytes": bbytes}
    else:
        res["bf16"] = {"us": float("nan")}
    # ragged batch of the same shape: sequence b attends to its first T_lens[b] positions
    # (seeded lengths in [T/4, T]); bytes are the packed records actually read. The padded
    # alternative is the uniform call at the longest length, masking nothing.
    if w.d == 128 and w.k_mode == 0 and w.v_mode == 0 and w.B <= 512:
        import random
        rnd = random.Random(1234)
        lens = [rnd.randint(w.T // 4, w.T) for _ in range(w.B)]
        per_tok = packed // (w.B * w.T)
        rbytes = sum(lens) * per_tok
        wsr = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, w.Hq, lens))
        rs = _time(lambda: tq.tq_decode_attention_varlen(q, cache, lens, w.scale, out, wsr, stream=stream),
                   stream, torch)
        wsp = tq.workspace(tq.tq_decode_workspace_bytes(cache, w.Hq, max(lens)))
        ps = _time(lambda: tq.tq_decode_attention(q, cache, max(lens), w.scale, out, wsp, stream=stream),
                   stream, torch)
        res["ragged"] = {"us": rs * 1e6, "gbs": rbytes / rs / 1e9, "frac": rbytes / rs / 1e9 / hbm,
                         "bytes": rbytes, "lengths": f"{w.B} sequences, seeded uniform in [T/4, T], "
                                                    f"min {min(lens)}, max {max(lens)}, sum {sum(lens)}",
                         "padded_uniform_us": ps * 1e6}
    # the same workload in a paged cache (64-position pages scattered over the pool by a
    # seeded permutation): bulk paged write, then paged decode over the full context
    if w.d == 128 and w.k_mode == 0 and w.v_mode == 0 and w.B <= 512 and K.dtype != torch.float32:
        page = 64
        maxp = (w.T + page - 1) // page
        npages = w.B * maxp
        g = torch.Generator().manual_seed(4321)
        bt = torch.randperm(npages, generator=g).to(torch.int32).reshape(w.B, maxp).cuda()
        pc = tq.TQPagedCache(w.B, w.Hkv, w.d, page, npages, maxp, w.k_bits, w.v_bits, bt, seed=cache.seed)
        tq.tq_quantize_kv_paged(K, V, pc, 0, stream=stream)
        lens = [w.T] * w.B
        wsp = tq.workspace(tq.tq_decode_paged_workspace_bytes(pc, w.Hq, lens))
        pgs = _time(lambda: tq.tq_decode_attention_paged(q, pc, lens, w.scale, out, wsp, stream=stream),
                    stream, torch)
        # the dense layout through the same per-sequence-length call, for comparison
        wsd = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, w.Hq, lens))
        dvs = _time(lambda: tq.tq_decode_attention_varlen(q, cache, lens, w.scale, out, wsd, stream=stream),
                    stream, torch)
        res["paged"] = {"us": pgs * 1e6, "gbs": packed / pgs / 1e9, "frac": packed / pgs / 1e9 / hbm,
                        "page_size": page, "layout": f"{npages} pages of {page} positions, scattered by a "
                                                     f"seeded permutation; every sequence at full length",
                        "dense_varlen_us": dvs * 1e6}
        del wsd
        del pc, bt, wsp
    # the pages' 3.5-bit operating point (4-bit keys, 3-bit values) on the same inputs
    if w.d == 128 and w.k_mode == 0 and w.v_mode == 0 and (w.k_bits, w.v_bits) != (4, 3):
        c35 = tq.TQCache(w.B, w.Hkv, w.T, w.d, 4, 3, seed=cache.seed)
        tq.tq_quantize_kv(K, V, c35, stream=stream)
        b35 = c35.packed_bytes(w.T)
        ws35 = tq.workspace(tq.tq_decode_workspace_bytes(c35, w.Hq, w.T))
        s35 = _time(lambda: tq.tq_decode_attention(q, c35, w.T, w.scale, out, ws35, stream=stream),
                    stream, torch)
        res["k4v3"] = {"us": s35 * 1e6, "gbs": b35 / s35 / 1e9, "frac": b35 / s35 / 1e9 / hbm,
                       "bytes": b35, "k": "4-bit MSE", "v": "3-bit MSE",
                       "reading": "3.5 bits per cached coordinate as 4-bit keys + 3-bit values"}
        del c35, ws35
    # end to end through the C ABI from pinned host buffers, as a serving loop runs it: every
    # step copies its inputs (query, the new token's K and V) in from pinned memory, runs the
    # two calls and reads its attention output back; the copies run on their own streams and
    # overlap the neighbouring steps' kernels (double-buffered device inputs and outputs).
    # Timed from the first copy-in to the last copy-out.
    hq = q.cpu().pin_memory()
    hk = k_new.cpu().pin_memory()
    hv = v_new.cpu().pin_memory()
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(q) for _ in range(2)]
    dk = [torch.empty_like(k_new) for _ in range(2)]
    dv = [torch.empty_like(v_new) for _ in range(2)]
    dout = [torch.empty_like(out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_read = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(s_in)
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i - 2])  # buffers j are free again
                dq[j].copy_(hq, non_blocking=True)
                dk[j].copy_(hk, non_blocking=True)
                dv[j].copy_(hv, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_read[i - 2])    # output j has been read back
            tq.tq_quantize_kv(dk[j], dv[j], cache, t_offset=w.T - 1, stream=stream)
            tq.tq_decode_attention(dq[j], cache, w.T, w.scale, dout[j], ws, stream=stream)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                hout[j].copy_(dout[j], non_blocking=True)
                ev_read[i].record(s_out)
        s_out.wait_stream(s_in)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n * 1e-3

    e2e_run(4)
    es = e2e_run(max(args.steps, 10))
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    res["e2e"] = {"value": packed / es / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": hout[0].numel() * hout[0].element_size(), "ms_per_step": es * 1e3,
                  "pipeline": "copy-in, compute and copy-out on three streams, double-buffered"}
    samples = {w.name: flip_sample(w, K, V, cache)}
    res["configs"] = {}
    for name in OTHER_WORKLOADS:
        if name == w.name:
            continue
        entry, sample = measure_workload(WORKLOADS_BY_NAME()[name], tq, torch, stream, hbm)
        res["configs"][name] = entry
        samples[name] = sample
        torch.cuda.empty_cache()
    res["prefill"] = measure_prefill(tq, torch, stream)
    # the oracle on the host cores (bounded sample), and the oracle's codes for the sampled
    # slice of every workload against the device's (the count of codes decided differently
    # near a decision boundary)
    if args.gpus == 1:
        res["cpu_baseline"] = time_oracle_decode(w)
        for name, sample in samples.items():
            flips = oracle_boundary_flips(*sample)
            if name == w.name:
                res["boundary_flips"] = flips
            else:
                res["configs"][name]["boundary_flips"] = flips
    return res


def measure_prefill(tq, torch, stream):
    """Chunked prefill attention over the compressed cache at long contexts (the
    Llama-3.1-8B shape, batch 4): a chunk of 1024 queries at the end of a 64K-token cache
    (4-bit keys, 2-bit values; also with the keys on the E2M1 grid) and of a 128K-token cache
    (3-bit keys and values). The roofline is
    the tensor cores': algorithmic FLOPs 4 d per (query row, visible key) against the measured
    dense bf16 peak."""
    import dataclasses

    from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs
    pk = tensor_peak()
    res = {}
    for label, name, T, kmode in (("64k", "llama3_8b_decode_32k", 65536, tq.TQ_MSE),
                                  ("128k", "llama3_8b_128k_3bit", 131072, tq.TQ_MSE),
                                  ("64k_e2m1_keys", "llama3_8b_decode_32k", 65536, tq.TQ_E2M1)):
        w = dataclasses.replace(WORKLOADS[name], B=4, T=T)
        Lq, t0 = 1024, T - 1024
        K, V, _ = make_inputs(w, device="cuda")
        cache = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, kmode, tq.TQ_MSE, seed=w.seed)
        tq.tq_quantize_kv(K, V, cache, stream=stream)
        del K, V
        g = torch.Generator(device="cuda").manual_seed(77)
        q = torch.randn(w.B, Lq, w.Hq, w.d, generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty(w.B, Lq, w.Hq, w.d, device="cuda")
        ts = _time(lambda: tq.tq_prefill_attention(q, cache, t0, w.scale, out, stream=stream), stream, torch,
                   min_calls=3, min_s=0.5)
        flops = w.B * w.Hq * 4 * w.d * (Lq * t0 + Lq * (Lq + 1) // 2)
        tf = flops / ts / 1e12
        res[label] = {"shape": f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d}, cache {T} positions, chunk Lq={Lq} at t0={t0}",
                      "k": f"{w.k_bits}-bit " + ("E2M1 (score MMAs on E2M1 operands)" if kmode == tq.TQ_E2M1 else "MSE"),
                      "v": f"{w.v_bits}-bit MSE", "us": ts * 1e6,
                      "tflops": tf, "peak_tflops": pk[0], "frac": tf / pk[0], "peak_source": pk[1],
                      "flops": flops, "flop_count": "4 d per (query row, visible cached key): q.k and p.v"}
        del cache, q, out
        torch.cuda.empty_cache()
    return res


def tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    return 1590.0, "fallback 1.59 PFLOP/s"


OTHER_WORKLOADS = ("tiny_single_head_fp32", "gpt2_prod_2bit", "llama3_8b_128k_3bit", "llama70b_asym_16k",
                   "llama3_8b_decode_32k")
FLIP_ROWS = 4096


def WORKLOADS_BY_NAME():
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS
    return WORKLOADS


def flip_sample(w, K, V, cache, n=FLIP_ROWS):
    """Inputs and device codes of the first n positions of (batch 0, KV head 0), K and V, as
    host arrays, for the count of boundary flips."""
    n = min(n, K.shape[2])
    out = [w, n]
    for side, X in (("k", K), ("v", V)):
        out.append(X[0, 0, :n].float().cpu().numpy())
        codes = cache[f"{side}_codes"]
        out.append(None if codes is None else codes[0, 0, :n].cpu().numpy())
        signs = cache[f"{side}_signs"]
        out.append(None if signs is None else signs[0, 0, :n].cpu().numpy())
    return tuple(out)


def oracle_boundary_flips(w, n, kx, kcodes, ksigns, vx, vcodes, vsigns):
    """CPU (oracle) leg: the oracle quantises the sampled rows in float64; device codes that
    differ from its codes are counted, with the number of coordinates within 1e-5 of a decision
    boundary (where the float32 device decision may legitimately differ) and, for
    TurboQuant_prod, sign bits that differ with |(S r)_j| < 1e-5 ||r||."""
    import numpy as np

    import oracle as O
    res = {}
    for side, x, codes, signs, bits, mode in (("k", kx, kcodes, ksigns, w.k_bits, w.k_mode),
                                              ("v", vx, vcodes, vsigns, w.v_bits, w.v_mode)):
        rec = O.quantize(x.astype(np.float64), bits, mode, seed=w.seed, qjl_seed=w.qjl_seed, m=w.qjl_m or None)
        wb = bits if mode == O.MSE else bits - 1
        near = O.boundary_distance(rec) < 1e-5
        if wb > 0:
            got = O.unpack_bits(codes, wb, w.d)
            diff = got != rec.codes
        else:
            diff = np.zeros_like(near)
        e = {"rows": int(n), "coords": int(near.size), "near_boundary": int(near.sum()),
             "flipped": int(diff.sum()), "flipped_away_from_boundary": int((diff & ~near).sum())}
        if mode == O.PROD:
            row_ok = ~np.any(diff, axis=1)
            gb = O.unpack_bits(signs, 1, rec.m)
            near_s = np.abs(rec.proj) < 1e-5 * rec.rnorm[:, None]
            bad = (gb != rec.qjl_bits) & row_ok[:, None]
            e["sign_bits"] = int(row_ok.sum() * rec.m)
            e["signs_flipped"] = int(bad.sum())
            e["signs_flipped_away_from_zero"] = int((bad & ~near_s).sum())
        res[side] = e
    return res


def measure_workload(w, tq, torch, stream, hbm):
    """One layer of workload w at full size: decode call (µs, GB/s, fraction of the HBM
    peak) and bulk quantise of the layer (µs, Mtok/s, fraction); for the 128K-context workload
    the 32-layer prefill write timed as one run; for the 70B-shaped one a bf16 boundary layer
    and the 80-layer decode step timed as one run."""
    from quantized_decode_attention_kv_b200.workloads import make_inputs
    K, V, q = make_inputs(w, device="cuda")
    cache = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, w.k_mode, w.v_mode, w.qjl_m,
                       w.qjl_m, seed=w.seed, qjl_seed=w.qjl_seed)
    tq.tq_quantize_kv(K, V, cache, stream=stream)
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, w.Hq, w.T))
    packed = cache.packed_bytes(w.T)
    dec = _time(lambda: tq.tq_decode_attention(q, cache, w.T, w.scale, out, ws, stream=stream), stream, torch)
    qt = _time(lambda: tq.tq_quantize_kv(K, V, cache, stream=stream), stream, torch, min_calls=20)
    qbytes = (K.numel() + V.numel()) * K.element_size() + packed
    e = {"shape": f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} T={w.T}",
         "k": f"{w.k_bits}-bit {'MSE' if w.k_mode == 0 else 'PROD'}",
         "v": f"{w.v_bits}-bit {'MSE' if w.v_mode == 0 else 'PROD'}",
         "decode_us": dec * 1e6, "decode_gbs": packed / dec / 1e9, "decode_frac": packed / dec / 1e9 / hbm,
         "packed_bytes": packed,
         "quantize_us": qt * 1e6, "quantize_mtok_s": w.B * w.T / qt / 1e6, "quantize_gbs": qbytes / qt / 1e9,
         "quantize_frac": qbytes / qt / 1e9 / hbm, "quantize_bytes": qbytes}
    sample = flip_sample(w, K, V, cache)
    if w.layers > 1 and not w.bf16_layers:
        # prefill write of every layer, timed as one run: layer l's K, V (two input buffers in
        # turn, each its own seeded draw) quantised into layer l's cache
        K2, V2, _ = make_inputs(w, device="cuda", layer=1)
        caches = [cache] + [tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, w.k_mode, w.v_mode,
                                       seed=w.seed) for _ in range(w.layers - 1)]
        ins = [(K, V), (K2, V2)]

        def write_all():
            for i, c in enumerate(caches):
                tq.tq_quantize_kv(*ins[i % 2], c, stream=stream)
        wt = _time(write_all, stream, torch, min_calls=3, min_s=0.5)
        e["prefill_write_all_layers"] = {
            "layers": w.layers, "us": wt * 1e6, "mtok_s": w.B * w.T / wt / 1e6,
            "gbs": w.layers * qbytes / wt / 1e9, "frac": w.layers * qbytes / wt / 1e9 / hbm,
            "bytes": w.layers * qbytes, "inputs": "two seeded input buffers used by alternate layers"}
        del caches, ins, K2, V2
    if w.bf16_layers:
        # a layer kept in bf16 (the same split-K design over the unquantised cache)
        wsb = tq.workspace(tq.tq_decode_bf16_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.d))
        bt = _time(lambda: tq.tq_decode_attention_bf16(q, K, V, w.T, w.scale, out, wsb, stream=stream),
                   stream, torch)
        bbytes = (K.numel() + V.numel()) * 2
        e["bf16_layer_decode"] = {"us": bt * 1e6, "gbs": bbytes / bt / 1e9, "frac": bbytes / bt / 1e9 / hbm,
                                  "bytes": bbytes}
        # the whole decode step over all layers: quantised layers write their new token and run
        # the compressed decode, bf16 layers run the bf16 decode over their own K, V
        layers = []
        for l in range(w.layers):
            Kl, Vl, ql = make_inputs(w, device="cuda", layer=l)
            if l in w.bf16_layers:
                layers.append(("bf16", Kl, Vl, ql, None))
            else:
                cl = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, seed=w.seed)
                tq.tq_quantize_kv(Kl, Vl, cl, stream=stream)
                layers.append(("tq", Kl[:, :, w.T - 1:].contiguous(), Vl[:, :, w.T - 1:].contiguous(), ql, cl))
                del Kl, Vl
        def step_all():
            for kind, a0, a1, ql, cl in layers:
                if kind == "bf16":
                    tq.tq_decode_attention_bf16(ql, a0, a1, w.T, w.scale, out, wsb, stream=stream)
                else:
                    tq.tq_quantize_kv(a0, a1, cl, t_offset=w.T - 1, stream=stream)
                    tq.tq_decode_attention(ql, cl, w.T, w.scale, out, ws, stream=stream)
        st = _time(step_all, stream, torch, min_calls=3, min_s=0.5)
        nq = w.layers - len(w.bf16_layers)
        sbytes = nq * packed + len(w.bf16_layers) * bbytes
        e["decode_step_all_layers"] = {
            "layers": w.layers, "bf16_layers": list(w.bf16_layers), "us": st * 1e6, "gbs": sbytes / st / 1e9,
            "frac": sbytes / st / 1e9 / hbm, "bytes": sbytes,
            "step": "per quantised layer: write of the new token + compressed decode; per bf16 layer: bf16 decode"}
        del layers
    del K, V, q, cache, ws
    return e, sample


def run_prefill_case(spec: str):
    """One prefill call on a stated case, for profilers (no timing, no JSON line)."""
    import dataclasses

    import torch

    from quantized_decode_attention_kv_b200 import tq
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs
    parts = spec.split(",")
    T, Lq = int(parts[0]), int(parts[1])
    kmode = tq.TQ_E2M1 if len(parts) > 2 and parts[2] == "e2m1" else tq.TQ_MSE
    w = dataclasses.replace(WORKLOADS[DEFAULT_WORKLOAD], B=4, T=T)
    K, V, _ = make_inputs(w, device="cuda")
    cache = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, kmode, tq.TQ_MSE, seed=w.seed)
    tq.tq_quantize_kv(K, V, cache)
    q = torch.randn(w.B, Lq, w.Hq, w.d, generator=torch.Generator(device="cuda").manual_seed(77),
                    device="cuda").to(torch.bfloat16)
    out = torch.empty(w.B, Lq, w.Hq, w.d, device="cuda")
    for _ in range(2):
        tq.tq_prefill_attention(q, cache, T - Lq, w.scale, out)
    torch.cuda.synchronize()
    print(json.dumps({"prefill_case": spec, "out_finite": bool(torch.isfinite(out).all())}))


def run_paged_case(T: int):
    """Two paged decode calls on a stated case, for profilers (no timing, no JSON line)."""
    import dataclasses

    import torch

    from quantized_decode_attention_kv_b200 import tq
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs
    w = dataclasses.replace(WORKLOADS[DEFAULT_WORKLOAD], T=T)
    K, V, q = make_inputs(w, device="cuda")
    page = 64
    maxp = (T + page - 1) // page
    bt = torch.randperm(w.B * maxp, generator=torch.Generator().manual_seed(4321)).to(torch.int32)
    pc = tq.TQPagedCache(w.B, w.Hkv, w.d, page, w.B * maxp, maxp, w.k_bits, w.v_bits,
                         bt.reshape(w.B, maxp).cuda(), seed=w.seed)
    tq.tq_quantize_kv_paged(K, V, pc, 0)
    lens = [T] * w.B
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_paged_workspace_bytes(pc, w.Hq, lens))
    for _ in range(2):
        tq.tq_decode_attention_paged(q, pc, lens, w.scale, out, ws)
    torch.cuda.synchronize()
    print(json.dumps({"paged_case": T, "out_finite": bool(torch.isfinite(out).all())}))


def main():
    args = parse_args()
    if args.paged_case:
        run_paged_case(args.paged_case)
        return
    if args.prefill_case:
        run_prefill_case(args.prefill_case)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
