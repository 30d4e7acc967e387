#!/usr/bin/env python
"""Benchmark of mixed-format paged decode attention on B200.

Workload (the long-context decode): 4 sequences x 131072 tokens, 24 query / 4 KV heads, head_dim
256, 48 layers' worth of pages in one pool (page 0 + the last 512 tokens + protected pages FP8,
about 96% of pages TQ3).  One step is one decode step of the whole 48-layer attention stack: for
every layer, append one new token per sequence (FP8), demote the pages leaving the 512-token
anchor window to TQ3, and run decode attention over the mixed cache.  Inputs are seeded
synthetic bf16 (``mixed_format_paged_mkv_b200.workloads``).  Every decode reads ~494 MB of pages
(> 126 MB L2) and the 48 layers cycle, so no L2 flush is needed.

Metric: decode-attention us/step and KV GB/s read.  ``value`` = algorithmic decode bytes of all
layers of all timed steps / device time of the steps (appends and demotions included in the
time), summed over ranks (replicas, weak scaling).  ``roofline`` is for the partial-attention
kernel, timed with CUDA events on its stream during the timed region.

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention µs/step and KV GB/s read (fraction of B200 HBM roofline)"
FALLBACK_HBM_GBS = 6650.0
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the partial-attention kernel, from
# the ncu capture summarised in profiles/, keyed by the hash of the kernel sources it measured.
NCU_TRAFFIC = {
    # profiles/decode_kernel_long_ctx128k_1layer.md: 494,519,552 B read + 4,348,928 B written
    # (re-keyed: since that capture only the D 64/128 launch bound changed; the captured
    # decode_kernel<256,1> is the same)
    "53ddc387bee37f97": 498868480,
}


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in ("decode.cu", "device_util.cuh", "mkv_internal.h"):
        with open(os.path.join(ROOT, "mixed_format_paged_mkv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------- byte accounting
def decode_bytes(tables, ctxs, Hkv, D, Hq, q_len):
    """Algorithmic bytes of one decode call over the given sequences:
    (total, partial-kernel share).  Per sequence: FP8 tokens x 2*Hkv*D + FP8 pages x 8*Hkv
    (scales) + TQ3 tokens x 0.875*Hkv*D + 4 B per table entry; plus q (bf16) and out (fp32)."""
    kv = 0.0
    ent = 0
    for t, L in zip(tables, ctxs):
        t = np.asarray(t, dtype=np.int64)
        fmt = t >> 30
        toks = np.full(t.size, 16, dtype=np.int64)
        toks[-1] = L - 16 * (t.size - 1)
        n8 = toks[fmt == 0].sum()
        p8 = int((fmt == 0).sum())
        n3 = toks[fmt == 1].sum()
        kv += n8 * 2 * Hkv * D + p8 * 8 * Hkv + n3 * 0.875 * Hkv * D
        ent += t.size
    q = len(ctxs) * q_len * Hq * D * 2
    out = len(ctxs) * q_len * Hq * D * 4
    return kv + 4 * ent + q + out, kv + q


# ---------------------------------------------------------------------------- ranks
def rank_max(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: float, world: int, elapsed_max_ms: float) -> float:
    """Whole-job GB/s of independent replicas: every rank's bytes over the slowest rank's time."""
    return bytes_per_rank * world / (elapsed_max_ms * 1e-3) / 1e9


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(w, seq=0, head=0, target_s=10.0, max_runs=None, warmup=0):
    """Time the CPU oracle's decode (dequantise the pages + float64 attention) of one sequence's
    one KV-head group over its full context.  Returns (GB/s, seconds per run, runs, cores, desc)."""
    from oracle import attention as A
    from oracle import formats as F
    from oracle import pool as P
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    L = w.lengths()[seq]
    k, v = w.kv(seq, 0)
    k, v = k[:, [head]], v[:, [head]]
    pool = P.RefPool(1, w.D, 1, -(-L // 16), -(-L // 16) + 1, -(-L // 16) + 1)
    pool.append([0], [L], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
    for p in w.protected(seq):
        pool.set_protected(0, p, 1)
    pool.demote([0], w.window)
    q = F.bf16_bits_to_f64(w.q(seq, 0))[:, head * w.g:(head + 1) * w.g]
    table = pool.block_table(0)
    total, _ = decode_bytes([table], [L], 1, w.D, w.g, w.q_len)

    def once():
        K, V = pool.dequant_seq(0)
        return A.attention(K, V, q, 1.0 / np.sqrt(w.D))

    for _ in range(warmup):
        once()
    times = []
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        once()
        times.append(time.perf_counter() - t0)
        if max_runs is not None and len(times) >= max_runs:
            break
        if max_runs is None and time.perf_counter() - t_start >= target_s:
            break
    per = sum(times) / len(times)
    desc = (f"decode of sequence {seq}, KV head {head} ({w.g} query heads) over {L} tokens "
            f"of layer 0: dequantise {len(table)} pages + float64 attention, {len(times)} runs")
    return total / per / 1e9, per, len(times), cores, desc


# ---------------------------------------------------------------------------- GPU arm
def build_pool(w, layers, extra_pages, device):
    import torch
    from mixed_format_paged_mkv_b200 import Pool
    pages = w.pages()
    n_prot = [len(w.protected(s)) for s in range(w.B)]
    anchors = [1 + w.window // 16 + 1 + n for n in n_prot]
    fp8 = max(max(pages) + sum(anchors), layers * sum(a + extra_pages for a in anchors)) + 64
    tq3 = layers * (sum(pages) + w.B * extra_pages) + 64
    pool = Pool(w.Hkv, w.D, w.B * layers, max(pages) + extra_pages, fp8, tq3, device=device)
    for fmt, n in ((0, fp8), (1, tq3)):
        order = w.slot_permutation(fmt, n)
        if order is not None:
            pool.set_slot_order(fmt, order)
    for op in w.build_ops(0):
        if op[0] == "append":
            k, v = w.kv(op[1], 0)
            kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).to(device)
            vt = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(device)
            pool.append([op[1]], [op[2]], kt, vt)
            del kt, vt
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, True)
        else:
            pool.demote([op[1]], op[2])
    for layer in range(1, layers):
        for s in range(w.B):
            pool.copy(s, layer * w.B + s)
    torch.cuda.synchronize()
    pool.device_status()
    return pool


def host_plan_us(pool, seq_ids, q_len, hq, reps=50):
    """Host time of planning one decode call (the work-unit cut), microseconds per call, measured
    after the timed region through the workspace query, which runs the same planner."""
    pool.workspace_bytes(seq_ids, q_len, hq)
    t0 = time.perf_counter()
    for _ in range(reps):
        pool.workspace_bytes(seq_ids, q_len, hq)
    return round((time.perf_counter() - t0) / reps * 1e6, 1)


def step_inputs_host(w, layers, steps, first_step):
    """[steps][layers] of (k, v, q) uint16 arrays stacked as k [S, Ly, B, Hkv, D] etc."""
    K = np.empty((steps, layers, w.B, w.Hkv, w.D), np.uint16)
    V = np.empty_like(K)
    Q = np.empty((steps, layers, w.B, w.q_len, w.Hq, w.D), np.uint16)
    for s in range(steps):
        for l in range(layers):
            K[s, l], V[s, l], Q[s, l] = w.step_inputs(first_step + s, l)
    return K, V, Q


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from mixed_format_paged_mkv_b200.workloads import WORKLOADS

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = WORKLOADS[4]
    layers = args.layers
    total_steps = args.warmup + args.steps + (args.warmup + args.steps if not args.no_e2e else 0)
    extra = total_steps // 16 + 3
    t_build = time.time()
    pool = build_pool(w, layers, extra, device)
    build_s = time.time() - t_build

    def as_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    seq_ids = [np.arange(l * w.B, (l + 1) * w.B, dtype=np.int32) for l in range(layers)]
    ones = np.ones(w.B, dtype=np.int32)
    n_dev = args.warmup + args.steps
    Kh, Vh, Qh = step_inputs_host(w, layers, n_dev, 0)
    Kd, Vd, Qd = as_bf16(Kh).to(device), as_bf16(Vh).to(device), as_bf16(Qh).to(device)
    outs = torch.empty((layers, w.B, w.q_len, w.Hq, w.D), dtype=torch.float32, device=device)
    ws_need = max(pool.workspace_bytes(seq_ids[0], w.q_len, w.Hq), 1 << 20)
    ws = torch.empty(int(ws_need * 1.5) + (1 << 20), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def one_step(Kt, Vt, Qt):
        for l in range(layers):
            pool.append(seq_ids[l], ones, Kt[l], Vt[l], stream=stream)
            pool.demote(seq_ids[l], w.window, stream=stream)
            pool.decode(seq_ids[l], Qt[l], out=outs[l], workspace=ws, stream=stream)

    def tables_now():
        tabs, ctxs = [], []
        for s in seq_ids[0]:
            t, L = pool.block_table(int(s))
            tabs.append(t)
            ctxs.append(L)
        return decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, w.q_len)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        return rank_max(x, world, device)

    # ---------------- device-resident run (value)
    for s in range(args.warmup):
        one_step(Kd[s], Vd[s], Qd[s])
    barrier()
    b0 = tables_now()
    launches0 = pool.launch_count()
    pool.timing(True)
    pool.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local_rank
    with ClockSampler(gpu_index) as clk:
        barrier()
        ev0.record(stream)
        for s in range(args.warmup, args.warmup + args.steps):
            one_step(Kd[s], Vd[s], Qd[s])
        ev1.record(stream)
        barrier()
    elapsed_ms = max_over_ranks(ev0.elapsed_time(ev1))
    tm = pool.timing_read()
    pool.timing(False)
    launches = pool.launch_count() - launches0
    b1 = tables_now()
    pool.device_status()
    per_call_total = 0.5 * (b0[0] + b1[0])
    per_call_partial = 0.5 * (b0[1] + b1[1])
    value_gbs = job_throughput(per_call_total * layers * args.steps, world, elapsed_ms)
    partial_ms = tm["partial_ms"] / max(tm["calls"], 1)
    achieved = per_call_partial / (partial_ms * 1e-3) / 1e9
    peak, peak_src = hbm_peak()

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        first = args.warmup + args.steps
        Kh2, Vh2, Qh2 = step_inputs_host(w, layers, args.warmup + args.steps, first)
        Kp = as_bf16(Kh2).pin_memory()
        Vp = as_bf16(Vh2).pin_memory()
        Qp = as_bf16(Qh2).pin_memory()
        Ks = torch.empty_like(Kd[0])
        Vs = torch.empty_like(Vd[0])
        Qs = torch.empty_like(Qd[0])
        out_h = torch.empty(outs.shape, dtype=torch.float32).pin_memory()
        h2d = (Ks.numel() + Vs.numel() + Qs.numel()) * 2
        d2h = out_h.numel() * 4

        def e2e_step(s):
            Ks.copy_(Kp[s], non_blocking=True)
            Vs.copy_(Vp[s], non_blocking=True)
            Qs.copy_(Qp[s], non_blocking=True)
            one_step(Ks, Vs, Qs)
            out_h.copy_(outs, non_blocking=True)

        for s in range(args.warmup):
            e2e_step(s)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.warmup, args.warmup + args.steps):
            e2e_step(s)
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1))
        b2 = tables_now()
        e2e_gbs = job_throughput(0.5 * (b1[0] + b2[0]) * layers * args.steps, world, e2e_ms)
        e2e = {"value": round(e2e_gbs, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms / args.steps, 4)}
        pool.device_status()

    res = {
        "metric": METRIC,
        "value": round(value_gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4),
        "us_per_layer_decode_step": round(1000 * elapsed_ms / args.steps / layers, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16xf16->f32 (e4m3 and 3-bit codes, exact f16 images)",
        "data": "synthetic (seeded bf16 N(0,1), 4 outlier K channels x8 per head)",
        "config": {"workload": w.name, "batch": w.B, "context": w.lengths()[0],
                   "layers": layers, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
                   "q_len": w.q_len, "anchor_window": w.window, "fp8_page_share": 0.04,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: each decode reads ~494 MB of pages; 48 layers cycle",
                   "decode_bytes_per_layer_call": int(per_call_total)},
        "roofline": {"bound": "hbm", "kernel": "decode_kernel (FP8 + TQ3 partial attention)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "traffic": NCU_TRAFFIC.get(kernel_hash()),
                     "bytes_per_launch": int(per_call_partial),
                     "launch_ms": round(partial_ms, 5),
                     "merge_ms": round(tm["merge_ms"] / max(tm["calls"], 1), 5)},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "build_s": round(build_s, 1),
        "host_plan_us_per_call": host_plan_us(pool, seq_ids[0], w.q_len, w.Hq),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, per, runs, cores, desc = oracle_sample(w, target_s=args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                               "kind": "oracle", "sample": desc,
                               "seconds_per_run": round(per, 3)}
    return res


def run_reference(args, rank, world):
    from mixed_format_paged_mkv_b200.workloads import WORKLOADS
    if rank != 0:
        return None
    w = WORKLOADS[4]
    gbs, per, runs, cores, desc = oracle_sample(w, max_runs=args.steps, warmup=args.warmup)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(gbs, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per * 1000, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded bf16 N(0,1), 4 outlier K channels x8 per head)",
        "config": {"workload": w.name, "batch": w.B, "context": w.lengths()[0], "layers": 48,
                   "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D, "q_len": w.q_len,
                   "parallelism": "host cores",
                   "step": "one bounded sample: " + desc},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- extra studies
# Measurements beyond the headline line, one JSON line per point (not part of the driver's
# contract): --mode sweep (FP8 page share from page 0 + window only up to all pages FP8, on one
# layer of the long-context workload), --mode canary (two 59,008-token sequences at the long
# workload's head shape, mixed cache against an all-FP8 control: decode time and KV bytes per
# token), --mode pack (bulk FP8 -> TQ3 demotion of an all-FP8 pool shaped like the batch-8
# workload, in GB/s), --mode prefill (direct bf16 -> TQ3 packing of that workload's prompts) and
# --mode materialise (dense fp32 K and V of that workload's sequences), --mode configs (decode
# µs per call, algorithmic GB/s and roofline fractions of every workload configuration, L2
# flushed before each call, and the steady-state append -> demote -> decode step).
def _bf16_tensor(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def _time_decode(pool, w, device, reps=20, warm=3):
    """Partial and merge time (µs) and algorithmic bytes of one decode call over all sequences
    of one layer, averaged over `reps` calls after `warm` untimed ones."""
    import torch
    seqs = list(range(w.B))
    q = _bf16_tensor(np.stack([w.q(s) for s in seqs]), device)
    out = torch.empty((w.B, w.q_len, w.Hq, w.D), dtype=torch.float32, device=device)
    ws = torch.empty(pool.workspace_bytes(seqs, w.q_len, w.Hq) + (1 << 20), dtype=torch.uint8,
                     device=device)
    for _ in range(warm):
        pool.decode(seqs, q, out=out, workspace=ws)
    torch.cuda.synchronize()
    pool.timing(True)
    pool.timing_read()
    for _ in range(reps):
        pool.decode(seqs, q, out=out, workspace=ws)
    tm = pool.timing_read()
    pool.timing(False)
    pool.device_status()
    tabs, ctxs = zip(*(pool.block_table(s) for s in seqs))
    total, partial = decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, w.q_len)
    n8 = sum(1 for t in tabs for e in t if (e >> 30) == 0)
    return dict(partial_us=1000 * tm["partial_ms"] / tm["calls"],
                merge_us=1000 * tm["merge_ms"] / tm["calls"], bytes=partial,
                fp8_page_share=n8 / sum(len(t) for t in tabs), out=out)


def run_extra(args):
    import torch
    from mixed_format_paged_mkv_b200 import Pool
    from mixed_format_paged_mkv_b200.workloads import WORKLOADS
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peak, peak_src = hbm_peak()
    lines = []
    if args.mode == "sweep":
        for frac in (0.0, 0.04, 0.25, 0.5, 1.0):
            w = WORKLOADS[4].scaled(fp8_page_frac=frac, layers=1)
            pool = build_pool(w, 1, 3, device)
            r = _time_decode(pool, w, device)
            gbs = r["bytes"] / (r["partial_us"] * 1e-6) / 1e9
            lines.append(dict(mode="sweep", workload=w.name, fp8_page_share=round(r["fp8_page_share"], 4),
                              partial_us=round(r["partial_us"], 2), merge_us=round(r["merge_us"], 2),
                              bytes_per_call=int(r["bytes"]), gbs=round(gbs, 1),
                              frac=round(gbs / peak, 4), peak_source=peak_src,
                              kv_bytes_per_token=round(pool.stats()[3], 1)))
            del pool
            torch.cuda.empty_cache()
    elif args.mode == "canary":
        res = {}
        for name, frac in (("mixed", 0.0), ("fp8_control", 1.0)):
            w = WORKLOADS[4].scaled(B=2, ctx=(59008, 59008), fp8_page_frac=frac, layers=1)
            pool = build_pool(w, 1, 3, device)
            r = _time_decode(pool, w, device)
            res[name] = dict(r, bpt=pool.stats()[3])
            del pool
            torch.cuda.empty_cache()
        m, c = res["mixed"], res["fp8_control"]
        diff = (m["out"] - c["out"]).abs().max().item()
        tm, tc = m["partial_us"] + m["merge_us"], c["partial_us"] + c["merge_us"]
        lines.append(dict(mode="canary", sequences=2, context=59008, q_heads=24, kv_heads=4, head_dim=256,
                          mixed_us=round(tm, 2), control_us=round(tc, 2),
                          throughput_vs_control=round(tc / tm, 4),
                          kv_bytes_per_token_mixed=round(m["bpt"], 1),
                          kv_bytes_per_token_control=round(c["bpt"], 1),
                          active_kv_ratio=round(c["bpt"] / m["bpt"], 4),
                          fp8_page_share_mixed=round(m["fp8_page_share"], 4),
                          max_abs_output_difference=diff))
    elif args.mode == "pack":
        w = WORKLOADS[2]
        pages = w.pages()
        n = sum(pages)
        pool = Pool(w.Hkv, w.D, 2 * w.B, max(pages) + 2, 2 * n + 64, n + 64, device=device)
        for s in range(w.B):  # templates: every page FP8
            k, v = w.kv(s, 0)
            pool.append([s], [w.lengths()[s]], _bf16_tensor(k, device), _bf16_tensor(v, device))
        torch.cuda.synchronize()
        work = list(range(w.B, 2 * w.B))
        stream = torch.cuda.current_stream()
        times, demoted = [], 0
        for rep in range(8):
            for s in range(w.B):
                pool.copy(s, w.B + s)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            demoted = pool.demote(work, w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
            for s in work:
                pool.reset(s)
        pool.device_status()
        per_page = w.Hkv * ((32 * w.D + 8) + 14 * w.D)
        ms = statistics.median(times)
        gbs = demoted * per_page / (ms * 1e-3) / 1e9
        lines.append(dict(mode="pack", workload=w.name, pages_demoted=demoted, bytes=demoted * per_page,
                          ms=round(ms, 4), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                          peak_source=peak_src,
                          note="one mkv_demote_pages call, host planning included in the span"))
    elif args.mode == "prefill":
        # direct bf16 -> TQ3 packing of the batch-8 workload's prompts (256-token window FP8)
        w = WORKLOADS[2]
        pages = w.pages()
        n = sum(pages)
        pool = Pool(w.Hkv, w.D, w.B, max(pages) + 2, n + 64, n + 64, device=device)
        ks, vs = zip(*(w.kv(s, 0) for s in range(w.B)))
        kd, vd = _bf16_tensor(np.concatenate(ks), device), _bf16_tensor(np.concatenate(vs), device)
        seqs, lens = list(range(w.B)), w.lengths()
        stream = torch.cuda.current_stream()
        times = []
        for rep in range(8):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            pool.prefill(seqs, lens, kd, vd, window=w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
            if rep < 7:
                for s in seqs:
                    pool.reset(s)
        pool.device_status()
        tabs = [pool.block_table(s)[0] for s in seqs]
        n3 = sum(1 for t in tabs for e in t if (e >> 30) == 1)
        n8 = sum(len(t) for t in tabs) - n3
        rd = sum(lens) * w.Hkv * w.D * 2 * 2
        wr = n3 * w.Hkv * 14 * w.D + n8 * w.Hkv * (32 * w.D + 16)
        ms = statistics.median(times)
        gbs = (rd + wr) / (ms * 1e-3) / 1e9
        lines.append(dict(mode="prefill", workload=w.name, tokens=sum(lens), tq3_pages=n3, fp8_pages=n8,
                          bytes=rd + wr, ms=round(ms, 4), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                          peak_source=peak_src,
                          note="one mkv_prefill_kv call (bf16 read, TQ3/FP8 pages written), host planning included"))
    elif args.mode == "materialise":
        w = WORKLOADS[2]
        pool = build_pool(w, 1, 3, device)
        L = max(w.lengths())
        k = torch.empty((L, w.Hkv, w.D), dtype=torch.float32, device=device)
        v = torch.empty_like(k)
        stream = torch.cuda.current_stream()
        for s in range(w.B):
            pool.materialise(s, k, v)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for rep in range(4):
            for s in range(w.B):
                pool.materialise(s, k, v)
        e1.record(stream)
        torch.cuda.synchronize()
        pool.device_status()
        tabs, ctxs = zip(*(pool.block_table(s) for s in range(w.B)))
        kv_bytes = decode_bytes(tabs, ctxs, w.Hkv, w.D, 0, 0)[1]
        out_bytes = sum(ctxs) * w.Hkv * w.D * 4 * 2
        ms = e0.elapsed_time(e1) / 4
        gbs = (kv_bytes + out_bytes) / (ms * 1e-3) / 1e9
        lines.append(dict(mode="materialise", workload=w.name, tokens=sum(ctxs), bytes=int(kv_bytes + out_bytes),
                          ms=round(ms, 4), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                          peak_source=peak_src, note="mkv_materialise_kv of every sequence (dense fp32 K and V)"))
    elif args.mode == "configs":
        from mixed_format_paged_mkv_b200.workloads import long_qlen4
        spec_tbs = 8.0  # the spec HBM figure, reported beside the measured peak
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)   # > 126 MB L2
        stream = torch.cuda.current_stream()
        for w in (WORKLOADS[1], WORKLOADS[2], WORKLOADS[3], WORKLOADS[4].scaled(layers=1),
                  long_qlen4().scaled(layers=1)):
            pool = build_pool(w, 1, 3, device)
            seqs = list(range(w.B))
            q = _bf16_tensor(np.stack([w.q(s) for s in seqs]), device)
            out = torch.empty((w.B, w.q_len, w.Hq, w.D), dtype=torch.float32, device=device)
            ws = torch.empty(pool.workspace_bytes(seqs, w.q_len, w.Hq) + (1 << 20),
                             dtype=torch.uint8, device=device)
            for _ in range(3):
                pool.decode(seqs, q, out=out, workspace=ws)
            pool.timing(True)
            pool.timing_read()
            for _ in range(20):   # L2 flushed before every call
                flush.zero_()
                pool.decode(seqs, q, out=out, workspace=ws)
            tm = pool.timing_read()
            pool.timing(False)
            pool.device_status()
            tabs, ctxs = zip(*(pool.block_table(s) for s in seqs))
            total, partial = decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, w.q_len)
            pu, mu = 1000 * tm["partial_ms"] / tm["calls"], 1000 * tm["merge_ms"] / tm["calls"]
            gbs = partial / (pu * 1e-6) / 1e9
            lines.append(dict(mode="configs", workload=w.name, sequences=w.B, tokens=int(sum(ctxs)),
                              q_len=w.q_len, partial_us=round(pu, 2), merge_us=round(mu, 2),
                              call_us=round(pu + mu, 2), algorithmic_bytes=int(total),
                              partial_gbs=round(gbs, 1), frac_of_measured=round(gbs / peak, 4),
                              frac_of_8tbs=round(gbs / (spec_tbs * 1000), 4),
                              call_gbs=round(total / ((pu + mu) * 1e-6) / 1e9, 1),
                              l2="flushed (256 MB write) before every call"))
            del pool, ws
            torch.cuda.empty_cache()
        # steady state: per step append 1 token per sequence, demote, decode
        w = WORKLOADS[5]
        warm, steps = 16, 64
        pool = build_pool(w, 1, (warm + steps) // 16 + 3, device)
        seqs = list(range(w.B))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(warm + steps)]
        out = torch.empty((w.B, 1, w.Hq, w.D), dtype=torch.float32, device=device)
        ws = torch.empty(int(pool.workspace_bytes(seqs, 1, w.Hq) * 1.5) + (1 << 20),
                         dtype=torch.uint8, device=device)
        ones = [1] * w.B
        demoted = 0
        kvq = [w.step_inputs(st, 0) for st in range(warm + steps)]
        kvq = [(_bf16_tensor(k, device), _bf16_tensor(v, device), _bf16_tensor(q, device))
               for k, v, q in kvq]
        for st in range(warm + steps):
            k, v, q = kvq[st]
            e = ev[st]
            e[0].record(stream)
            pool.append(seqs, ones, k, v)
            e[1].record(stream)
            n = pool.demote(seqs, w.window)
            e[2].record(stream)
            pool.decode(seqs, q, out=out, workspace=ws)
            e[3].record(stream)
            if st >= warm:
                demoted += n
        torch.cuda.synchronize()
        pool.device_status()
        ph = np.array([[ev[st][i].elapsed_time(ev[st][i + 1]) for i in range(3)]
                       for st in range(warm, warm + steps)]) * 1000
        tabs, ctxs = zip(*(pool.block_table(s) for s in seqs))
        total, partial = decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, 1)
        dec = float(np.median(ph[:, 2]))
        lines.append(dict(mode="configs", workload=w.name, sequences=w.B, tokens=int(sum(ctxs)),
                          steps=steps, append_us=round(float(np.median(ph[:, 0])), 2),
                          demote_us=round(float(np.median(ph[:, 1])), 2), decode_us=round(dec, 2),
                          step_us=round(float(np.median(ph.sum(1))), 2),
                          pages_demoted_per_step=round(demoted / steps, 2),
                          decode_call_gbs=round(total / (dec * 1e-6) / 1e9, 1),
                          frac_of_measured=round(total / (dec * 1e-6) / 1e9 / peak, 4),
                          note="medians over the timed steps; spans include host planning"))
    for l in lines:
        print(json.dumps(l), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--mode", choices=["bench", "sweep", "canary", "pack", "prefill", "materialise",
                                       "configs"],
                    default="bench",
                    help="extra studies on one GPU (one JSON line per point); default: the bench")
    args = ap.parse_args()
    if args.mode != "bench":
        run_extra(args)
        return
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch.distributed as dist
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_gpu(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
