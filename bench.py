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
PROFILES = os.path.join(ROOT, "profiles")


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in ("decode.cu", "decode_partial.cuh", "decode_d64.cu", "decode_d128.cu",
              "decode_d256.cu", "device_util.cuh", "mkv_internal.h"):
        with open(os.path.join(ROOT, "mixed_format_paged_mkv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of `kernel` from the ncu summaries
    under profiles/: a summary states it on a line
    ``traffic_bytes_per_launch: <kernel> <bytes> sources <hash>``, where <hash> is kernel_hash() of
    the sources that were captured.  None when no summary matches the current sources."""
    want = kernel_hash()
    try:
        names = sorted(os.listdir(PROFILES))
    except OSError:
        return None
    for n in names:
        if not n.endswith((".md", ".txt")):
            continue
        with open(os.path.join(PROFILES, n)) as f:
            for line in f:
                parts = line.strip().strip("`").split()
                if (len(parts) == 5 and parts[0] == "traffic_bytes_per_launch:" and
                        parts[1] == kernel and parts[3] == "sources" and parts[4] == want):
                    return int(parts[2])
    return None


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
        fmt = (t >> 30) & 3
        toks = np.full(t.size, 16, dtype=np.int64)
        toks[-1] = L - 16 * (t.size - 1)
        n8 = toks[fmt == 0].sum()
        p8 = int((fmt == 0).sum())
        n3 = toks[fmt == 1].sum()
        n16 = toks[fmt == 2].sum()          # BF16 control pages
        kv += n8 * 2 * Hkv * D + p8 * 8 * Hkv + n3 * 0.875 * Hkv * D + n16 * 4 * Hkv * D
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
    """SM clock and clock-event reasons of one GPU, sampled every `period` seconds by a host
    thread through NVML queries while the block runs (read only: no setting is changed).
    Falls back to `nvidia-smi -lms` when NVML is not importable."""
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period: float = 0.005):
        self.device_index = device_index
        self.period = period
        self.samples = []
        self.max_mhz = None
        self.source = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _loop(self, h):
        import pynvml
        reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = reason_fn(h)
                self.samples.append((sm, r))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self.thread = None
        self.proc = None
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._loop, args=(h,), daemon=True)
            self.thread.start()
            self.source = f"nvml every {self.period * 1000:.0f} ms"
        except Exception:
            fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.sw_power_cap,"
                      "clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                      "clocks_event_reasons.hw_thermal_slowdown")
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                     "-lms", "20", "-i", str(self.device_index)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi every 20 ms"
                time.sleep(0.3)
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            names = ["sw_power_cap", "hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown"]
            for l in out.splitlines():
                f = [x.strip() for x in l.split(",")]
                try:
                    mask = sum(self.REASONS[n] for n, v in zip(names, f[2:6]) if v.lower() == "active")
                    self.samples.append((float(f[0]), mask))
                    self.max_mhz = float(f[1])
                except (ValueError, IndexError):
                    continue

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = sorted(n for n, bit in self.REASONS.items()
                         if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples),
                "sm_min_mhz": min(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": self.source}


# ---------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(w, seq=0, head=0, target_s=10.0, max_runs=None, warmup=0, threads=None):
    """Time the CPU oracle's decode (dequantise the pages + float64 attention) of one sequence's
    one KV-head group over its full context, with its BLAS limited to `threads` (None: all the
    host's cores).  Returns (GB/s, seconds per run, runs, threads used, desc)."""
    from threadpoolctl import threadpool_info, threadpool_limits

    from oracle import attention as A
    from oracle import formats as F
    from oracle import pool as P
    limiter = threadpool_limits(limits=threads)
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
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
    limiter.restore_original_limits()
    per = sum(times) / len(times)
    desc = (f"decode of sequence {seq}, KV head {head} ({w.g} query heads) over {L} tokens "
            f"of layer 0: dequantise {len(table)} pages + float64 attention, {len(times)} runs")
    return total / per / 1e9, per, len(times), cores, desc


# ---------------------------------------------------------------------------- GPU arm
def build_pool(w, layers, extra_pages, device, bf16_control=False):
    import torch
    from mixed_format_paged_mkv_b200 import Pool
    pages = w.pages()
    n_prot = [len(w.protected(s)) for s in range(w.B)]
    anchors = [1 + w.window // 16 + 1 + n for n in n_prot]
    fp8 = max(max(pages) + sum(anchors), layers * sum(a + extra_pages for a in anchors)) + 64
    tq3 = layers * (sum(pages) + w.B * extra_pages) + 64
    if bf16_control:      # every page stays in the first slab as BF16
        fp8, tq3 = layers * (sum(pages) + w.B * extra_pages) + 64, 0
    pool = Pool(w.Hkv, w.D, w.B * layers, max(pages) + extra_pages, fp8, tq3, device=device,
                bf16_control=bf16_control)
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
    # three timed passes (value, kernel share, end to end) after their warm-ups append tokens
    n_dev = args.warmup + 2 * args.steps
    total_steps = n_dev + (args.warmup + args.steps if not args.no_e2e else 0)
    extra = total_steps // 16 + 3
    t_build = time.time()
    pool = build_pool(w, layers, extra, device)
    build_s = time.time() - t_build

    def as_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    seq_ids = [np.arange(l * w.B, (l + 1) * w.B, dtype=np.int32) for l in range(layers)]
    ones = np.ones(w.B, dtype=np.int32)
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

    def timed(first):
        """Steps [first, first + steps) between two events on the stream; returns ms."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record(stream)
        for s in range(first, first + args.steps):
            one_step(Kd[s], Vd[s], Qd[s])
        e1.record(stream)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    # ---------------- pass 1: the headline, no per-call instrumentation
    for s in range(args.warmup):
        one_step(Kd[s], Vd[s], Qd[s])
    barrier()
    b0 = tables_now()
    launches0 = pool.launch_count()
    with ClockSampler(local_rank) as clk:
        elapsed_ms = timed(args.warmup)
    launches = pool.launch_count() - launches0
    b1 = tables_now()
    pool.device_status()
    per_call_total = 0.5 * (b0[0] + b1[0])
    value_gbs = job_throughput(per_call_total * layers * args.steps, world, elapsed_ms)

    # ---------------- pass 2: the same steps with the library's per-call kernel events (three
    # per decode call, on the stream the kernels run on) for the partial-attention kernel's time
    pool.timing(True)
    pool.timing_read()
    instrumented_ms = timed(args.warmup + args.steps)
    tm = pool.timing_read()
    pool.timing(False)
    b2 = tables_now()
    pool.device_status()
    per_call_partial = 0.5 * (b1[1] + b2[1])
    partial_ms = tm["partial_ms"] / max(tm["calls"], 1)
    achieved = per_call_partial / (partial_ms * 1e-3) / 1e9
    peak, peak_src = hbm_peak()

    # ---------------- pass 3: end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        first = n_dev
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
        b3 = tables_now()
        e2e_gbs = job_throughput(0.5 * (b2[0] + b3[0]) * layers * args.steps, world, e2e_ms)
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
        "dtype": "f16 MMA, f32 accumulate (e4m3 and 3-bit codes, exact f16 images)",
        "data": "synthetic (seeded bf16 N(0,1), 4 outlier K channels x8 per head)",
        "config": {"workload": w.name, "batch": w.B, "context": w.lengths()[0],
                   "layers": layers, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
                   "q_len": w.q_len, "anchor_window": w.window, "fp8_page_share": 0.04,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: each decode reads ~494 MB of pages; 48 layers cycle",
                   "decode_bytes_per_layer_call": int(per_call_total)},
        "roofline": {"bound": "hbm", "kernel": "partial_kernel: the FP8 and TQ3 grids of a call",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "traffic": ncu_traffic("partial_grids"),
                     "bytes_per_launch": int(per_call_partial),
                     "launch_ms": round(partial_ms, 5),
                     "merge_ms": round(tm["merge_ms"] / max(tm["calls"], 1), 5),
                     "timed": "second pass of the same steps with per-call events on the stream",
                     "instrumented_ms_per_step": round(instrumented_ms / args.steps, 4)},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "build_s": round(build_s, 1),
        "host_plan_us_per_call": host_plan_us(pool, seq_ids[0], w.q_len, w.Hq),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, per, runs, cores, desc = oracle_sample(w, target_s=args.cpu_seconds)
        gbs1, per1, _, _, _ = oracle_sample(w, target_s=args.cpu_seconds / 2, threads=1)
        res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                               "kind": "oracle", "sample": desc,
                               "seconds_per_run": round(per, 3),
                               "single_thread": {"value": round(gbs1, 4), "unit": "GB/s",
                                                 "cores": 1, "seconds_per_run": round(per1, 3)}}
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


_FLUSH = None


def _flush_l2(device):
    """Write a buffer twice the size of the 126 MB L2, so the next call reads its pages from HBM."""
    global _FLUSH
    import torch
    if _FLUSH is None:
        _FLUSH = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    _FLUSH.zero_()


def _time_decode(pool, w, device, reps=20, warm=3):
    """Partial and merge time (µs) and algorithmic bytes of one decode call over all sequences
    of one layer, averaged over `reps` calls after `warm` untimed ones; L2 is flushed before
    every call (the library's per-call events exclude the flush)."""
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
        _flush_l2(device)
        pool.decode(seqs, q, out=out, workspace=ws)
    tm = pool.timing_read()
    pool.timing(False)
    pool.device_status()
    tabs, ctxs = zip(*(pool.block_table(s) for s in seqs))
    total, partial = decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, w.q_len)
    n8 = sum(1 for t in tabs for e in t if ((e >> 30) & 3) != 1)
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
    elif args.mode == "ablation":
        # one grid per page format (default) against one fused grid, on the long-context layer
        # and on the FP8-share sweep points
        for frac in (0.0, 0.04, 0.25, 1.0):
            w = WORKLOADS[4].scaled(fp8_page_frac=frac, layers=1)
            pool = build_pool(w, 1, 3, device)
            for fused in (False, True):
                pool.set_decode_kernels(fused)
                r = _time_decode(pool, w, device)
                gbs = r["bytes"] / (r["partial_us"] * 1e-6) / 1e9
                lines.append(dict(mode="ablation", kernels="fused" if fused else "split",
                                  workload=w.name, fp8_page_share=round(r["fp8_page_share"], 4),
                                  partial_us=round(r["partial_us"], 2),
                                  merge_us=round(r["merge_us"], 2),
                                  bytes_per_call=int(r["bytes"]), gbs=round(gbs, 1),
                                  frac=round(gbs / peak, 4), peak_source=peak_src))
            del pool
            torch.cuda.empty_cache()
    elif args.mode == "profile":
        # a small target for ncu: one layer of the long-context workload, a few decode calls
        w = WORKLOADS[4].scaled(layers=1, q_len=args.q_len,
                                name=WORKLOADS[4].name + ("" if args.q_len == 1 else f"_q{args.q_len}"))
        pool = build_pool(w, 1, 3, device)
        pool.set_decode_kernels(args.fused)
        seqs = list(range(w.B))
        q = _bf16_tensor(np.stack([w.q(s) for s in seqs]), device)
        out = torch.empty((w.B, w.q_len, w.Hq, w.D), dtype=torch.float32, device=device)
        ws = torch.empty(pool.workspace_bytes(seqs, w.q_len, w.Hq) + (1 << 20), dtype=torch.uint8,
                         device=device)
        for _ in range(args.steps):
            pool.decode(seqs, q, out=out, workspace=ws)
        torch.cuda.synchronize()
        pool.device_status()
        tabs, ctxs = zip(*(pool.block_table(s) for s in seqs))
        total, partial = decode_bytes(tabs, ctxs, w.Hkv, w.D, w.Hq, w.q_len)
        lines.append(dict(mode="profile", workload=w.name, calls=args.steps,
                          partial_bytes_per_call=int(partial), kernel_sources=kernel_hash()))
    elif args.mode == "canary":
        # two 59,008-token decodes at the long workload's head shape: the mixed cache against
        # an all-FP8 control and a BF16 control (pages stored as bf16), L2 flushed before every
        # timed call of every arm
        res = {}
        for name, frac, ctl in (("mixed", 0.0, False), ("fp8_control", 1.0, False),
                                ("bf16_control", 0.0, True)):
            w = WORKLOADS[4].scaled(B=2, ctx=(59008, 59008), fp8_page_frac=frac, layers=1)
            pool = build_pool(w, 1, 3, device, bf16_control=ctl)
            r = _time_decode(pool, w, device)
            res[name] = dict(r, bpt=pool.stats()[3])
            del pool
            torch.cuda.empty_cache()
        m = res["mixed"]
        tm = m["partial_us"] + m["merge_us"]
        line = dict(mode="canary", sequences=2, context=59008, q_heads=24, kv_heads=4, head_dim=256,
                    mixed_us=round(tm, 2), kv_bytes_per_token_mixed=round(m["bpt"], 1),
                    fp8_page_share_mixed=round(m["fp8_page_share"], 4),
                    l2="flushed (256 MB write) before every timed call of every arm")
        for name in ("fp8_control", "bf16_control"):
            c = res[name]
            tc = c["partial_us"] + c["merge_us"]
            line.update({f"{name}_us": round(tc, 2),
                         f"throughput_vs_{name}": round(tc / tm, 4),
                         f"kv_bytes_per_token_{name}": round(c["bpt"], 1),
                         f"active_kv_ratio_vs_{name}": round(c["bpt"] / m["bpt"], 4),
                         f"max_abs_output_difference_vs_{name}":
                             (m["out"] - c["out"]).abs().max().item()})
        lines.append(line)
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
        times, dev_times = [], []
        for rep in range(8):
            for s in range(w.B):
                pool.copy(s, w.B + s)
            torch.cuda.synchronize()
            # call span: host planning and launches included
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            demoted = pool.demote(work, w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
            for s in work:
                pool.reset(s)
            for s in range(w.B):
                pool.copy(s, w.B + s)
            torch.cuda.synchronize()
            # device time only: a spin kernel keeps the GPU busy while the host plans
            torch.cuda._sleep(20_000_000)
            e0.record(stream)
            pool.demote(work, w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                dev_times.append(e0.elapsed_time(e1))
            for s in work:
                pool.reset(s)
        pool.device_status()
        per_page = w.Hkv * ((32 * w.D + 8) + 14 * w.D)
        ms, dms = statistics.median(times), statistics.median(dev_times)
        gbs, dgbs = demoted * per_page / (ms * 1e-3) / 1e9, demoted * per_page / (dms * 1e-3) / 1e9
        lines.append(dict(mode="pack", workload=w.name, pages_demoted=demoted, bytes=demoted * per_page,
                          ms=round(ms, 4), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                          device_ms=round(dms, 4), device_gbs=round(dgbs, 1),
                          device_frac=round(dgbs / peak, 4), peak_source=peak_src,
                          note="one mkv_demote_pages call: ms is the call span with host "
                               "planning, device_ms the device work alone"))
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
        times, dev_times = [], []
        for rep in range(8):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            pool.prefill(seqs, lens, kd, vd, window=w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
            for s in seqs:
                pool.reset(s)
            torch.cuda._sleep(20_000_000)
            e0.record(stream)
            pool.prefill(seqs, lens, kd, vd, window=w.window)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                dev_times.append(e0.elapsed_time(e1))
            if rep < 7:
                for s in seqs:
                    pool.reset(s)
        pool.device_status()
        tabs = [pool.block_table(s)[0] for s in seqs]
        n3 = sum(1 for t in tabs for e in t if (e >> 30) == 1)
        n8 = sum(len(t) for t in tabs) - n3
        rd = sum(lens) * w.Hkv * w.D * 2 * 2
        wr = n3 * w.Hkv * 14 * w.D + n8 * w.Hkv * (32 * w.D + 16)
        ms, dms = statistics.median(times), statistics.median(dev_times)
        gbs, dgbs = (rd + wr) / (ms * 1e-3) / 1e9, (rd + wr) / (dms * 1e-3) / 1e9
        lines.append(dict(mode="prefill", workload=w.name, tokens=sum(lens), tq3_pages=n3, fp8_pages=n8,
                          bytes=rd + wr, ms=round(ms, 4), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                          device_ms=round(dms, 4), device_gbs=round(dgbs, 1),
                          device_frac=round(dgbs / peak, 4), peak_source=peak_src,
                          note="one mkv_prefill_kv call (bf16 read, TQ3/FP8 pages written): ms is "
                               "the call span with host planning, device_ms the device work alone"))
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
    ap.add_argument("--fused", action="store_true", help="--mode profile: the fused kernel")
    ap.add_argument("--q-len", type=int, default=1, help="--mode profile: new tokens per sequence")
    ap.add_argument("--mode", choices=["bench", "sweep", "canary", "pack", "prefill", "materialise",
                                       "configs", "ablation", "profile"],
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
