"""Benchmark of the MLA paged-KV decode hot path on B200.

One step = the whole hot path over one batch: split-KV schedule
(mla_get_metadata) + decode kernel + split-KV combine (mla_decode_fwd), all
through the C ABI.  Inputs are resident in HBM before the timed region; L2 is
flushed (256 MiB write) before every timed step and each step is timed with
CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
  python bench.py --op append [--workload NAME]   (the cache-append kernel, see run_append)
  python bench.py --trace [--workload NAME] [--batch B]   (per-phase cycles, trace build)

Prints ONE JSON line on rank 0.  By default the line's top-level numbers are
those of the FP8 656-byte-cache workload (b=128, h_q=128, L ~ U[16384, 32768],
the compute-bound configuration) in TFLOP/s, and `per_config` holds the same
record for the four other workloads.  For each workload:
  value        algorithmic flops / (time of the K timed steps / K); a step
               replays a CUDA graph of schedule + decode + combine
  roofline     the decode call alone (decode + combine kernels), median of at
               least 50 calls each after an L2 flush, against the measured
               peak of the bound (tensor or HBM)
  e2e          through the public API with inputs uploaded from pinned host
               memory and results downloaded every step
  cpu_baseline the float64 oracle on the host cores, bounded sample
Under torchrun each rank runs an independent replica of the workloads
(requests are independent, there is no data-path collective); the time is the
max over ranks and `value` aggregates all ranks.  `--impl reference` times the
float64 CPU oracle on a bounded sample instead.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MLA decode TFLOPS & effective HBM GB/s on 1 B200 (frac of roofline)"
# the arithmetic the tensor cores run on for each cache format
MMA = {"bf16": "bf16 operands, fp32 accumulation",
       "fp8_656": "bf16 operands (FP8 cache dequantised to bf16 in shared memory), fp32 accumulation"}
DTYPE = {"bf16": "bf16", "fp8_656": "bf16"}
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# ---------------------------------------------------------------------------
# algorithmic work (what the method must move / compute)
# ---------------------------------------------------------------------------

def algorithmic_work(w: W.Workload, seqlens: np.ndarray):
    """Bytes and flops of one pass, counting valid tokens and visible pairs only.

    bytes = sum_b L_b * T  (T = 1152 bf16 / 656 fp8 per token)
          + |q| + |out| + |lse| + 4 * sum_b ceil(L_b / 64) (block-table reads) + 4 b (seqlens)
    flops = 2 * (576 + 512) * h_q * sum over (request, query token) of visible keys
    """
    T = 1152 if w.fmt == "bf16" else 656
    L = seqlens.astype(np.int64)
    B = L.size
    kv = int(L.sum()) * T
    q = B * w.s_q * w.h_q * 576 * 2
    out = B * w.s_q * w.h_q * 512 * 2
    lse = B * w.s_q * w.h_q * 4
    meta = 4 * int(((L + 63) // 64).sum()) + 4 * B
    vis = 0
    for i in range(w.s_q):
        vis += int(np.clip(L - w.s_q + i + 1, 0, None).sum()) if w.causal else int(L.sum())
    flops = 2 * (576 + 512) * w.h_q * vis
    return dict(bytes=kv + q + out + lse + meta, kv_bytes=kv, flops=flops)


def sparse_work(w: W.Workload, seqlens: np.ndarray, indices: np.ndarray):
    """Bytes and flops of one sparse decode: every valid list entry (0 <= idx < L)
    is one key read (656 bytes) and one (query token, key) pair per head.

    bytes = 656 * valid + |q| + |out| + |lse| + 4 * |indices| + 4 * valid
            (block-table entries) + 4 b (lengths)
    flops = 2 * (576 + 512) * h_q * valid
    """
    L = seqlens.astype(np.int64)[:, None, None]
    valid = int(((indices >= 0) & (indices < L)).sum())
    B = L.shape[0]
    q = B * w.s_q * w.h_q * 576 * 2
    out = B * w.s_q * w.h_q * 512 * 2
    lse = B * w.s_q * w.h_q * 4
    nbytes = 656 * valid + q + out + lse + 4 * indices.size + 4 * valid + 4 * B
    return dict(bytes=nbytes, kv_bytes=656 * valid, flops=2 * (576 + 512) * w.h_q * valid)


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("decode.cu", "sm100.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "mla_paged_kv_04_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes (read + write) of one decode launch from the committed ncu
    record, or None if there is none for this workload or the kernel source
    changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == workload and parts[1] == sha:
                return int(parts[2]) + int(parts[3])
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        self.proc = None
        self.gpu = gpu_index

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={CLOCK_QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        loaded = [s for s in sm if smax and s >= 0.3 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# the CPU oracle as a timed baseline (bounded sample)
# ---------------------------------------------------------------------------

def oracle_threads() -> int:
    """Threads the oracle's numpy BLAS runs with (what `cores` reports)."""
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_rate(w: W.Workload, budget_s: float = 12.0, seed: int = 0):
    """Time the float64 oracle on whole requests of the workload until `budget_s`.

    The sample is fixed: four single requests drawn with the workload's
    recipe (seeds seed .. seed + 3), cycled in order; one untimed call first
    (page faults of the first allocation).  Returns ({"tflops", "gbs"} of
    algorithmic work per second of oracle time, sample description, BLAS
    threads).
    """
    import oracle
    pool = []
    for b in range(4):
        one = W.Workload(w.name, 1, w.s_q, w.h_q, w.seqlen, fmt=w.fmt, causal=w.causal, seed=seed + b, topk=w.topk)
        case = W.make_case(one, poison=False)
        a = W.oracle_arrays(case)
        if w.topk:
            a["indices"] = case["indices"].numpy()
            work = sparse_work(one, a["cache_seqlens"], a["indices"])
        else:
            work = algorithmic_work(one, a["cache_seqlens"])
        pool.append((a, work["bytes"], work["flops"]))

    def call(a):
        if w.topk:
            oracle.mla_sparse_decode(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                                     a["indices"], a["softmax_scale"])
        else:
            oracle.mla_decode(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                              a["softmax_scale"], a["causal"])

    call(pool[0][0])
    n_done, t_total, bytes_done, flops_done = 0, 0.0, 0, 0
    while t_total < budget_s and n_done < 4096:
        a, nbytes, nflops = pool[n_done % len(pool)]
        t0 = time.perf_counter()
        call(a)
        t_total += time.perf_counter() - t0
        bytes_done += nbytes
        flops_done += nflops
        n_done += 1
    sample = (f"{n_done} whole requests of {w.describe()} cycled from 4 drawn with seeds {seed}..{seed + 3} "
              f"({t_total:.1f} s of oracle time)")
    return ({"tflops": flops_done / t_total / 1e12, "gbs": bytes_done / t_total / 1e9}, sample,
            oracle_threads())


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job rate: the units all ranks processed per second of the slowest
    rank's time (weak scaling: every rank runs its own replica)."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    """The reference arm: the float64 oracle on the host cores, on the same
    workload, metric and unit as the CUDA arm's line, each step a bounded
    sample of whole requests.  Rank 0 only."""
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload or HEADLINE]
    per_step, gbs = [], []
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    sample = ""
    cores = oracle_threads()
    for i in range(args.warmup + args.steps):
        rate, sample, cores = oracle_rate(w, budget_s=budget, seed=0)
        if i >= args.warmup:
            per_step.append(rate["tflops"])
            gbs.append(rate["gbs"])
    value = statistics.mean(per_step)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.describe(), "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q,
                       "seqlen": list(w.seqlen), "kv_format": w.fmt},
            "gbs": statistics.mean(gbs),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {sample}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


HEADLINE = "fp8_656"          # the compute-bound configuration (FP8 656-byte cache)
PER_CONFIG = ["tiny", "uniform_bf16", "varlen_spec_bf16", "long_ctx_bf16", "sparse_fp8"]
MIN_REPS = 50                 # decode calls timed for the roofline, at least (a short burst: a
                              # loop of seconds runs into the power cap and measures that instead)


def measure_workload(w: W.Workload, args, world, rank, dev, peaks, cpu_budget: float, sampler_gpu: int):
    """Everything bench.py reports for one workload on this rank.

    Returns (record, total_ms_of_the_K_steps) where record holds the rank's
    numbers; the caller takes the max over ranks of the step time.
    """
    import mla_paged_kv_04_b200 as mla
    case = W.make_case(w, seed=w.seed + rank, device=dev, poison=False)
    q, kv, bt, L = case["q"], case["kv_cache"], case["block_table"], case["cache_seqlens"]
    B, s_q, h_q = case["batch"], w.s_q, w.h_q
    parts = args.parts or mla.mla_default_num_sm_parts(dev)
    sched = torch.empty(mla.mla_metadata_size(B, s_q, h_q, parts) // 4, dtype=torch.int32, device=dev)
    ns = torch.empty(mla.mla_num_splits_len(B, s_q, h_q), dtype=torch.int32, device=dev)
    ws = mla.alloc_workspace(B, s_q, h_q, parts, dev)
    out = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    seqlens_np = L.cpu().numpy()
    stream = torch.cuda.current_stream(dev)
    if w.topk:
        # the sparse decode over the same kind of cache: its own schedule and workspace
        idx = case["indices"]
        work = sparse_work(w, seqlens_np, idx.cpu().numpy())
        sched = torch.empty(mla.mla_sparse_metadata_size_bytes(B, s_q, h_q, parts) // 4, dtype=torch.int32,
                            device=dev)
        ns = torch.empty(mla.mla_sparse_num_splits_len(B, s_q, h_q), dtype=torch.int32, device=dev)
        ws = torch.zeros(mla.mla_sparse_workspace_size(B, s_q, h_q, parts), dtype=torch.uint8, device=dev)

        def meta(st=stream):
            mla.mla_get_sparse_metadata(B, s_q, h_q, w.topk, parts, device=dev, sched=sched, num_splits=ns,
                                        stream=st)

        def decode(st=stream):
            mla.mla_sparse_decode_fwd(q, kv, bt, L, idx, w.softmax_scale, sched, ns, parts, out, lse, ws, stream=st)
    else:
        work = algorithmic_work(w, seqlens_np)

        def meta(st=stream):
            mla.mla_get_metadata(L, s_q, h_q, parts, sched=sched, num_splits=ns, stream=st)

        def decode(st=stream):
            mla.mla_decode_fwd(q, kv, w.fmt, bt, L, w.softmax_scale, w.causal, sched, ns, parts, out, lse, ws,
                               stream=st)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        meta()
        decode()
    torch.cuda.synchronize(dev)
    status = mla.mla_last_device_status(ws)
    if status != 0:
        raise SystemExit(f"{w.name}: device status {mla.STATUS.get(status, status)} during warm-up")

    reps = max(MIN_REPS, args.steps)

    # The calls are replayed from CUDA graphs, captured once through the
    # public API: a step's kernels then reach the GPU back to back, and the
    # event pair measures the GPU's time, not the host's launch overhead
    # (for small batches the host is slower than the kernels).  The L2 flush
    # runs before each timed step, outside the graph and the event pair.
    #   g_step: schedule + decode + combine (one step of the hot path)
    #   g_call: decode + combine (the decode call, for the roofline)
    #   g_meta: the schedule alone
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    g_step, g_call, g_meta = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    meta_c = lambda: meta(cap)
    decode_c = lambda: decode(cap)
    with torch.cuda.stream(cap):
        meta_c()
        decode_c()
    cap.synchronize()
    with torch.cuda.graph(g_step, stream=cap):
        meta_c()
        decode_c()
    with torch.cuda.graph(g_call, stream=cap):
        decode_c()
    with torch.cuda.graph(g_meta, stream=cap):
        meta_c()
    stream.wait_stream(cap)
    for _ in range(3):
        flush.zero_()
        g_step.replay()
    torch.cuda.synchronize(dev)

    # The timed steps: one event pair per step around the whole hot path
    # (schedule + decode + combine), L2 flushed before each.  No event sits
    # between the kernels, so the decode kernel's programmatic early launch
    # overlaps the schedule kernel's tail as it would in a serving loop.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    dec_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    meta_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(MIN_REPS)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(sampler_gpu) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            g_step.replay()
            ev[i][1].record(stream)
        # The decode call alone (decode + combine kernels), for the roofline:
        # the median of `reps` calls, each after an L2 flush and the schedule.
        for i in range(reps):
            flush.zero_()
            g_meta.replay()
            dec_ev[i][0].record(stream)
            g_call.replay()
            dec_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    dec_ms = [e[0].elapsed_time(e[1]) for e in dec_ev]
    for i in range(MIN_REPS):  # the schedule kernel alone
        flush.zero_()
        meta_ev[i][0].record(stream)
        g_meta.replay()
        meta_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    meta_ms = [e[0].elapsed_time(e[1]) for e in meta_ev]
    del g_step, g_call, g_meta
    status = mla.mla_last_device_status(ws)
    if status != 0:
        raise SystemExit(f"{w.name}: device status {mla.STATUS.get(status, status)} in the timed region")

    # End to end through the public API: every step uploads its inputs (q,
    # block table, sequence lengths) from pinned host memory, flushes L2, runs
    # the schedule and the decode, and downloads its results (out, lse); the
    # paged KV cache is resident state.  Steps are pipelined two deep on three
    # streams, as a serving loop runs them: step i+1's upload and step i-1's
    # download overlap step i's kernels (double-buffered inputs and outputs).
    # The timed region runs from the first upload to the last download of the
    # K timed steps.
    q_h = q.cpu().pin_memory()
    bt_h = bt.cpu().pin_memory()
    L_h = L.cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    lse_h = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    q_d = [torch.empty_like(q) for _ in range(2)]
    bt_d = [torch.empty_like(bt) for _ in range(2)]
    L_d = [torch.empty_like(L) for _ in range(2)]
    out_d = [out, torch.empty_like(out)]
    lse_d = [lse, torch.empty_like(lse)]
    h2d = q_h.numel() * 2 + bt_h.numel() * 4 + L_h.numel() * 4
    if w.topk:
        idx_h = idx.cpu().pin_memory()
        idx_d = [torch.empty_like(idx) for _ in range(2)]
        h2d += idx_h.numel() * 4
    d2h = out_h[0].numel() * 2 + lse_h[0].numel() * 4
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    dn_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        k = i % 2
        with torch.cuda.stream(s_up):
            s_up.wait_event(cmp_done[k])  # step i - 2 has read buffer k
            q_d[k].copy_(q_h, non_blocking=True)
            bt_d[k].copy_(bt_h, non_blocking=True)
            L_d[k].copy_(L_h, non_blocking=True)
            if w.topk:
                idx_d[k].copy_(idx_h, non_blocking=True)
            up_done[k].record(s_up)
        stream.wait_event(up_done[k])
        stream.wait_event(dn_done[k])  # step i - 2's results have left buffer k
        flush.zero_()
        if w.topk:
            mla.mla_get_sparse_metadata(B, s_q, h_q, w.topk, parts, device=dev, sched=sched, num_splits=ns,
                                        stream=stream)
            mla.mla_sparse_decode_fwd(q_d[k], kv, bt_d[k], L_d[k], idx_d[k], w.softmax_scale, sched, ns, parts,
                                      out_d[k], lse_d[k], ws, stream=stream)
        else:
            mla.mla_get_metadata(L_d[k], s_q, h_q, parts, sched=sched, num_splits=ns, stream=stream)
            mla.mla_decode_fwd(q_d[k], kv, w.fmt, bt_d[k], L_d[k], w.softmax_scale, w.causal, sched, ns, parts,
                               out_d[k], lse_d[k], ws, stream=stream)
        cmp_done[k].record(stream)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(cmp_done[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            lse_h[k].copy_(lse_d[k], non_blocking=True)
            dn_done[k].record(s_dn)

    for i in range(max(args.warmup, 3)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_up)
    w0 = max(args.warmup, 3)
    for i in range(w0, w0 + args.steps):
        e2e_step(i)
    e_end.record(s_dn)
    torch.cuda.synchronize(dev)
    e2e_total = max_over_ranks(e_start.elapsed_time(e_end), world)
    status = mla.mla_last_device_status(ws)
    if status != 0:
        raise SystemExit(f"{w.name}: device status {mla.STATUS.get(status, status)} in the end-to-end steps")

    n = world
    ms_per_step = total_ms / args.steps
    dec_med = statistics.median(dec_ms)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if work["flops"] / work["bytes"] > ridge:
        ach = work["flops"] / (dec_med * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"]}
    else:
        ach = work["bytes"] / (dec_med * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"]}
    roof.update({"traffic": recorded_traffic(w.name) if args.batch is None else None,
                 "kernel": "decode (+ split-KV combine) via mla_decode_fwd",
                 "peak_source": f"{peaks['source']} (burst)", "algorithmic_bytes": work["bytes"],
                 "algorithmic_flops": work["flops"], "median_ms": dec_med, "reps": reps,
                 "min_ms": min(dec_ms), "tflops": work["flops"] / (dec_med * 1e-3) / 1e12,
                 "gbs": work["bytes"] / (dec_med * 1e-3) / 1e9})
    e2e_ms = e2e_total / args.steps
    cpu = None
    if world == 1 and cpu_budget > 0:
        rate, sample, cores = oracle_rate(w, budget_s=cpu_budget)
        cpu = {"value": rate["tflops"], "unit": "TFLOP/s", "gbs": rate["gbs"], "cores": cores, "kind": "oracle",
               "sample": sample}
    rec = {
        "workload": w.describe(), "value": aggregate_rate(work["flops"], ms_per_step, n) / 1e12,
        "unit": "TFLOP/s", "gbs": aggregate_rate(work["bytes"], ms_per_step, n) / 1e9,
        "ms_per_step": ms_per_step, "metadata_ms": statistics.median(meta_ms),
        "config": {"workload": w.describe(), "batch": B, "s_q": w.s_q, "h_q": w.h_q, "seqlen": list(w.seqlen),
                   "kv_format": w.fmt, "causal": w.causal, "num_sm_parts": parts, "mma": MMA[w.fmt]},
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": n * work["flops"] / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "gbs": n * work["bytes"] / (e2e_ms * 1e-3) / 1e9,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "uploads, kernels (with the L2 flush) and downloads of consecutive steps "
                              "overlap on three streams, two buffers deep"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    del case, q, kv, bt, L, ws, out, lse, flush, q_d, bt_d, L_d, out_d, lse_d
    torch.cuda.empty_cache()
    return rec


def run_cuda(args, world, rank, local):
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    mla.load_library()
    dev = torch.device("cuda", local if world > 1 else 0)
    peaks = load_peaks()
    head = W.WORKLOADS[args.workload or HEADLINE]
    if args.batch is not None:
        head = dataclasses.replace(head, batch=args.batch)
    others = [] if (args.workload or args.batch is not None) else [W.WORKLOADS[n] for n in PER_CONFIG]
    cpu_head = 0.0 if args.no_cpu_baseline else args.cpu_budget
    cpu_other = 0.0 if args.no_cpu_baseline else min(3.0, args.cpu_budget)
    rec = measure_workload(head, args, world, rank, dev, peaks, cpu_head, dev.index or 0)
    per = {}
    for w in others:
        per[w.name] = measure_workload(w, args, world, rank, dev, peaks, cpu_other, dev.index or 0)
    if rank != 0:
        return
    n = world
    line = {
        "metric": METRIC, "value": rec["value"], "unit": rec["unit"], "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE[head.fmt], "data": "synthetic",
        "config": dict(rec["config"], **{
            "launch": "each timed step replays a CUDA graph of the public calls (schedule, decode, combine)",
            "l2": "flushed before every timed step and every roofline rep (256 MiB write)",
            "parallelism": f"replicas x{n} (independent request batches)"}),
        "gbs": rec["gbs"],
        "metadata_ms": rec["metadata_ms"],
        "roofline": rec["roofline"],
        "cpu_baseline": rec["cpu_baseline"],
        "e2e": rec["e2e"],
        "gpu_launches": rec["gpu_launches"],
        "clocks": rec["clocks"],
        "per_config": per,
    }
    print(json.dumps(line), flush=True)


def run_trace(args):
    """One decode call of the workload through the trace build; prints the
    median length of each pipeline phase in SM cycles (and saves the raw
    timestamps with --trace-out)."""
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import build, trace
    build.build(trace=True)
    mla.load_library(trace=True)
    w = W.WORKLOADS[args.workload or HEADLINE]
    if args.batch is not None:
        w = dataclasses.replace(w, batch=args.batch)
    dev = torch.device("cuda", 0)
    case = W.make_case(w, device=dev, poison=False)
    q, kv, bt, L = case["q"], case["kv_cache"], case["block_table"], case["cache_seqlens"]
    B = case["batch"]
    parts = args.parts or mla.mla_default_num_sm_parts(dev)
    out = torch.empty((B, w.s_q, w.h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, w.s_q, w.h_q), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if w.topk:
        sched, ns = mla.mla_get_sparse_metadata(B, w.s_q, w.h_q, w.topk, parts, device=dev)
        ws = torch.zeros(mla.mla_sparse_workspace_size(B, w.s_q, w.h_q, parts), dtype=torch.uint8, device=dev)
    else:
        sched, ns = mla.mla_get_metadata(L, w.s_q, w.h_q, parts)
        ws = mla.alloc_workspace(B, w.s_q, w.h_q, parts, dev)

    def run():
        flush.zero_()
        if w.topk:
            mla.mla_sparse_decode_fwd(q, kv, bt, L, case["indices"], w.softmax_scale, sched, ns, parts, out, lse, ws)
        else:
            mla.mla_decode_fwd(q, kv, w.fmt, bt, L, w.softmax_scale, w.causal, sched, ns, parts, out, lse, ws)

    for _ in range(3):
        run()
    ts = trace.record(run)
    status = mla.mla_last_device_status(ws)
    if args.trace_out:
        np.save(args.trace_out, ts)
    print(f"# {w.describe()}, {parts} CTA pairs, device status {mla.STATUS.get(status, status)}")
    print(trace.format_summary(trace.summarize(ts)))


# ---------------------------------------------------------------------------
# the cache-append kernel (mla_kv_append)
# ---------------------------------------------------------------------------

APPEND_METRIC = "KV-cache append effective HBM GB/s on 1 B200 (frac of roofline)"
APPEND_TOKENS = 2048  # new tokens per request in the timed append (a chunk of prefill)


def append_work(fmt: str, batch: int, s_new: int) -> int:
    """Algorithmic bytes of one append: the new bf16 rows read, the cache rows
    written (1,152 or 656 bytes), one block-table entry per token, the lengths."""
    tokens = batch * s_new
    return tokens * (1152 + (1152 if fmt == "bf16" else 656)) + 4 * tokens + 4 * batch


def oracle_append_rate(w: W.Workload, budget_s: float = 5.0):
    """The oracle's append on whole-page chunks of new tokens until `budget_s`."""
    import oracle
    case = W.make_case(w, seqlens=[256], poison=False)
    a = W.oracle_arrays(case)
    g = torch.Generator().manual_seed(7)
    new = torch.randn((1, 64, 576), generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle.append_tokens(a["kv_cache"], w.fmt, new, a["block_table"], a["cache_seqlens"])
        n += 1
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return (append_work(w.fmt, 1, 64) * n / dt / 1e9, f"{n} appends of 64 new tokens into one "
            f"{w.fmt} request ({dt:.1f} s of oracle time)", cores)


def run_append(args, world, rank, local):
    """Time mla_kv_append: APPEND_TOKENS new tokens into every request of the
    workload's cache (the last APPEND_TOKENS positions), L2 flushed before each
    step; also a decode step's append (s_q new tokens per request)."""
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    mla.load_library()
    w = W.WORKLOADS[args.workload or HEADLINE]
    dev = torch.device("cuda", local if world > 1 else 0)
    case = W.make_case(w, seed=w.seed + rank, device=dev, poison=False)
    kv, bt, L = case["kv_cache"], case["block_table"], case["cache_seqlens"]
    B = w.batch
    s_new = min(APPEND_TOKENS, int(L.min().item()))
    gen = torch.Generator(device=dev).manual_seed(1000 + rank)
    new = torch.randn((B, s_new, 576), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    step_new = new[:, -w.s_q:].contiguous()  # a decode step's new tokens
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    work = append_work(w.fmt, B, s_new)

    for _ in range(args.warmup):
        flush.zero_()
        mla.mla_kv_append(new, kv, w.fmt, bt, L, ws, stream=stream)
        mla.mla_kv_append(step_new, kv, w.fmt, bt, L, ws, stream=stream)
    torch.cuda.synchronize(dev)
    status = mla.mla_last_device_status(ws)
    if status != 0:
        raise SystemExit(f"device status {mla.STATUS.get(status, status)} during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index or 0) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            mla.mla_kv_append(new, kv, w.fmt, bt, L, ws, stream=stream)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    small_ms = []
    for i in range(args.steps):
        flush.zero_()
        e1, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e1.record(stream)
        mla.mla_kv_append(step_new, kv, w.fmt, bt, L, ws, stream=stream)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        small_ms.append(e1.elapsed_time(e2))
    # end to end through the public call: upload the new tokens from pinned
    # memory, append, read the status word back
    new_h = new.cpu().pin_memory()
    st_h = torch.empty(4, dtype=torch.uint8).pin_memory()
    new_d = torch.empty_like(new)
    barrier(world)
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for i in range(args.steps):
        new_d.copy_(new_h, non_blocking=True)
        mla.mla_kv_append(new_d, kv, w.fmt, bt, L, ws, stream=stream)
        st_h.copy_(ws[:4], non_blocking=True)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world) / args.steps
    status = mla.mla_last_device_status(ws)
    if status != 0:
        raise SystemExit(f"device status {mla.STATUS.get(status, status)} in the timed region")
    if rank != 0:
        return
    peaks = load_peaks()
    n = world
    ms_per_step = total_ms / args.steps
    achieved = work / (statistics.mean(step_ms) * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs, sample, cores = oracle_append_rate(w)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample}
    line = {
        "metric": APPEND_METRIC, "value": aggregate_rate(work, ms_per_step, n) / 1e9, "unit": "GB/s", "n_gpus": n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.fmt == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": f"append into {w.describe()}", "op": "append", "batch": B, "s_new": s_new,
                   "kv_format": w.fmt, "l2": "flushed before every timed step (256 MiB write)",
                   "parallelism": f"replicas x{n} (independent request batches)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "append_kernel",
                     "peak_source": peaks["source"], "algorithmic_bytes": work},
        "decode_step_append_us": 1000 * statistics.median(small_ms),
        "cpu_baseline": cpu,
        "e2e": {"value": n * work / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": new.numel() * 2,
                "d2h_bytes_per_step": 4, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=list(W.WORKLOADS),
                    help=f"measure only this workload (default: {HEADLINE} as the headline, "
                         f"the others under per_config)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling runs)")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--parts", type=int, default=0, help="CTA pairs (default: SMs / 2)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="decode", choices=["decode", "append"])
    ap.add_argument("--trace", action="store_true", help="per-tile phase timings from the trace build")
    ap.add_argument("--trace-out", default=None, help="with --trace: save the raw timestamps (.npy)")
    args = ap.parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    if args.trace:
        run_trace(args)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        (run_append if args.op == "append" else run_cuda)(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
