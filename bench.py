"""Benchmark of the HiLS-Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hils|reference] [--quick]

Headline (`value`): prefill throughput in tokens/s on the prefill workload (B4 T8192 Hq16 Hkv4 d128
S64 k16 W512, bf16). One step = one pass of the prefill hot path over the batch: landmark summaries
(hils_chunk_summary), retrieval + GQA top-k (hils_select_topk) and Eq. 10 attention (hils_attn_fwd),
inputs resident in HBM, L2 flushed (a 256 MiB write) between timed steps and outside the events.
The same JSON line carries the decode workload (B8, 512K-token cache, 256 steps in a CUDA graph,
us/token), the context-length sweep, the training step (forward + backward, B2 T8192), a roofline
object per block, the end-to-end number through the public API with host buffers, the oracle's CPU
time on a bounded sample, and the SM clocks sampled during the timed region.

Multi-GPU (torchrun, one process per GPU): the batch is independent across sequences, so every rank
runs its own batch (different seed) with no data-path collective: weak scaling; `value` = tokens of
all ranks / max over ranks of the device time.
--impl reference times the fp64 CPU oracle (the reference arm for this method) on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunk_wise_hierarchical_summary_b200 import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index), "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:  # no nvidia-smi: the line carries no clock record
            self.proc = None
            if self.path is not None and os.path.exists(self.path):
                os.unlink(self.path)
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarise_clocks(lines)


def summarise_clocks(lines):
    """Summary of nvidia-smi CSV rows (no header, no units) in ClockSampler.FIELDS order: the median SM
    clock, the maximum SM clock, the throttle reasons seen active in any row, and the row count; None
    without a complete row."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return None
    sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
            "reasons": reasons, "samples": len(rows)}


class Dist:
    def __init__(self, n_gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local_rank])
            else:
                self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = torch.device("cuda", self.local_rank) if torch.cuda.is_available() else torch.device("cpu")
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def weak_scaling_value(dist: Dist, ms_local: float, units_per_rank: float):
    """Whole-job throughput under weak scaling: every rank processes `units_per_rank` independent units
    (its own sequences; no data-path collective), and the job takes as long as its slowest rank.
    Returns (max-over-ranks milliseconds, units per second over all ranks)."""
    ms = dist.max(ms_local)
    return ms, dist.world * units_per_rank / (ms / 1e3)


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic inputs: ranks draw distinct sequences of the same shapes."""
    return base + rank


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].strip().isdigit():
            return int(ids[local_rank])
    return local_rank


def timed_steps(steps, fn_stages, warmup, flush, dist: Dist, sampler=None):
    """Run `warmup` untimed steps, then `steps` timed ones. fn_stages() launches one step and returns
    nothing; stage boundaries are marked by the callback `mark` it receives. Returns per-stage device
    milliseconds summed over the timed steps (list) and the total."""
    for _ in range(warmup):
        fn_stages(lambda: None)
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()
    dist.barrier()
    if sampler:
        sampler.start()
    records = []
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True)]
        evs[0].record()

        def mark():
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            evs.append(e)

        fn_stages(mark)
        records.append(evs)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop() if sampler else None
    n_stage = len(records[0]) - 1
    stage_ms = [sum(r[i].elapsed_time(r[i + 1]) for r in records) for i in range(n_stage)]
    return stage_ms, sum(stage_ms), clocks


# ----------------------------------------------------------------------------- the line both arms print

METRIC = ("HiLS prefill tokens/s (B4 T8192 Hq16 Hkv4 d128 S64 k16 W512); decode us/token at 512K ctx in 'decode'; "
          "% of TC/HBM roofline")


# DRAM bytes (read + write) of one attn_tc_kernel launch at the prefill workload, from one ncu capture
# (`--metrics dram__bytes_read.sum,dram__bytes_write.sum` of `bench.py --profile attn`), or None when the
# kernel has changed since that capture. The last capture (241.7 MB read, 102.2 MB written: the inputs
# read once) predates the kernel's launch order across (batch, KV group), so the line reports None.
ATTN_TC_TRAFFIC_BYTES = None
ATTN_TC_LAST_CAPTURE_BYTES = 241742336 + 102183680


def base_config(w: W.Workload, world: int) -> dict:
    """The workload both arms report (identical dicts, so the two lines name the same configuration)."""
    return {"workload": w.name, "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": f"dp{world} (independent sequences per GPU)",
            "l2": "flushed (256 MiB write) between timed prefill steps, outside the events"}


# ----------------------------------------------------------------------------- algorithmic work

def window_left(p, Wn, S):
    return (max(0, p - Wn + 1) // S) * S


def prefill_work(w: W.Workload):
    """Algorithmic flops of the prefill hot path and of each stage, from the sizes alone.
    attention: 4 d flops per (query row, head, attended token) (QK^T and PV), attended = window + selected
    chunk tokens; routing: 2 d per (row, head, candidate chunk); summaries: 4 S d per (head, chunk)."""
    attended = 0
    cand = 0
    for p in range(w.q_pos0, w.q_pos0 + w.T):
        l = window_left(p, w.W, w.S)
        n = l // w.S
        attended += (p - l + 1) + min(w.topk, n) * w.S
        cand += n
    rows = w.B * w.Hq
    attn = 4 * w.d * attended * rows
    route = 2 * w.d * cand * rows
    summ = 4 * w.S * w.d * w.Nc * w.B * w.Hq
    el = 2 if w.dtype == "bf16" else 4
    attn_bytes = el * (w.B * w.Hq * w.T * w.d * 3 + w.B * w.Hkv * w.L * w.d * 2) + 4 * w.B * w.Hq * w.T \
        + (el * w.d + 4) * w.B * w.Hq * w.Nc
    return {"attn_flops": attn, "route_flops": route, "summary_flops": summ, "attn_bytes": attn_bytes,
            "avg_attended": attended / w.T}


def decode_bytes(w: W.Workload, idx=None):
    """Bytes one decode step must touch for its M = w.T queries at the end of the cache: every candidate
    summary once (k' in the input dtype + fp32 b'; the last query's candidates, the most), the K and V
    of the selected chunks and of the window, and q, q^ and the output. With M > 1 the queries of a
    KV group share what they touch: chunks count once per group over the union of the M selections
    (`idx` [B, Hkv, M, topk] of one step; without it, the per-query sum is an upper bound) and the
    window is the union of the M windows, tokens l_(L-M) .. L-1."""
    el = 2 if w.dtype == "bf16" else 4
    M = w.T
    p_last = w.L - 1
    n_last = window_left(p_last, w.W, w.S) // w.S
    summ = w.B * w.Hq * n_last * (w.d * el + 4)
    tile = w.S * w.d * el * 2
    if M > 1 and idx is not None:
        ids = idx.reshape(w.B * w.Hkv, M * w.topk).cpu()
        chunks = sum(len(set(r.tolist()) - {-1}) for r in ids) * tile
    else:
        chunks = sum(w.B * w.Hkv * min(w.topk, window_left(w.L - M + m, w.W, w.S) // w.S) * tile
                     for m in range(M))
    win = w.B * w.Hkv * (w.L - window_left(w.L - M, w.W, w.S)) * w.d * el * 2
    io = w.B * w.Hq * M * (w.d * el * 3 + 4)
    return {"total": summ + chunks + win + io, "summaries": summ, "chunks": chunks, "window": win, "io": io}


# ----------------------------------------------------------------------------- GPU arms

def bench_prefill(args, dist, dev, H, peaks):
    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=rank_seed(1000, dist.rank), device=dev)
    k_sum = torch.empty((w.B, w.Hq, w.Nc, w.d), dtype=torch.bfloat16, device=dev)
    b_sum = torch.empty((w.B, w.Hq, w.Nc), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.Hkv, w.T, w.topk), dtype=torch.int32, device=dev)
    shat = torch.empty((w.B, w.Hq, w.T, w.topk), dtype=torch.float32, device=dev)
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(mark):
        H.chunk_summary(x["k"], x["q_land"], w.S, k_sum=k_sum, b_sum=b_sum)
        mark()
        H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W, idx=idx,
                      shat=shat)
        mark()
        H.attn_fwd_shat(x["q"], x["k"], x["v"], idx, shat, S=w.S, window=w.W, out=out, lse=lse)
        mark()

    sampler = ClockSampler(physical_gpu_index(dist.local_rank))
    stage_ms, total_ms, clocks = timed_steps(args.steps, step, args.warmup, flush, dist, sampler)
    work = prefill_work(w)
    attn_s = stage_ms[2] / args.steps / 1e3
    achieved = work["attn_flops"] / attn_s / 1e12
    # union ratio of the selections (chunks a 32-query tile must visit / chunks each query selects)
    res = {
        "workload": w, "x": x, "out": out, "lse": lse, "idx": idx, "stage_ms": [s / args.steps for s in stage_ms],
        "ms_per_step": total_ms / args.steps, "clocks": clocks, "work": work,
        "roofline": {"bound": "tensor", "kernel": "hils_attn_fwd_shat (attn_tc_kernel)", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": ATTN_TC_TRAFFIC_BYTES,
                     "note": "algorithmic flops = 4*d per (row, head, attended token); attended = window + "
                             "selected chunk tokens, %.1f per query on average; traffic = DRAM bytes per "
                             "attn_tc_kernel launch (ncu)%s" % (
                                 work["avg_attended"], "" if ATTN_TC_TRAFFIC_BYTES is not None else
                                 ", null: the kernel's launch order changed after its last capture (%.1f MB per "
                                 "launch, the inputs read once)" % (ATTN_TC_LAST_CAPTURE_BYTES / 1e6))},
        "launches_per_step": 3,
    }
    del flush
    return res


def bench_prefill_e2e(args, dist, dev, H, res):
    """Same metric through the public API with host buffers: every step copies the inputs from pinned
    host memory, runs the prefill calls and copies out + lse back. The sequences of the batch are
    independent, so the step is pipelined per sequence over two streams: sequence b's copies back to
    the host overlap sequence b+1's copies in and its kernels (PCIe is full duplex)."""
    w = res["workload"]
    xh = {n: res["x"][n].cpu().pin_memory() for n in ("q", "k", "v", "q_hat", "q_land")}
    xd = {n: torch.empty_like(res["x"][n]) for n in xh}
    out_h = torch.empty(res["out"].shape, dtype=res["out"].dtype).pin_memory()
    lse_h = torch.empty(res["lse"].shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in xh.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * 4
    steps = max(1, min(args.steps, 10))
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]

    def step(mark):
        cur = torch.cuda.current_stream(dev)
        start = torch.cuda.Event()
        start.record(cur)
        for s in streams:
            s.wait_event(start)
        for b in range(w.B):
            s = streams[b % 2]
            with torch.cuda.stream(s):
                for n in xh:
                    xd[n][b].copy_(xh[n][b], non_blocking=True)
                sl = slice(b, b + 1)
                out, lse, _, _, _ = H.prefill(xd["q"][sl], xd["k"][sl], xd["v"][sl], xd["q_hat"][sl],
                                              xd["q_land"][sl], S=w.S, topk=w.topk, window=w.W)
                out_h[b].copy_(out[0], non_blocking=True)
                lse_h[b].copy_(lse[0], non_blocking=True)
        for s in streams:
            cur.wait_stream(s)
        mark()

    _, total_ms, _ = timed_steps(steps, step, 2, None, dist)
    ms, value = weak_scaling_value(dist, total_ms / steps, w.B * w.T)
    return {"value": value, "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "public API (prefill per sequence), pinned host buffers, copies pipelined over two streams"}


def bench_decode(args, dist, dev, H, peaks, w: W.Workload, steps: int):
    x = W.decode_inputs(w, seed=rank_seed(2000, dist.rank), device=dev)
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    # the cache's summaries (stage (a)), timed once more on their own: K + landmark queries in, k' + b' out
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    H.chunk_summary(x["k_cache"], x["q_land"], w.S, k_sum=k_sum, b_sum=b_sum)
    e1.record()
    torch.cuda.synchronize()
    summ_ms = e0.elapsed_time(e1)
    el = 2 if w.dtype == "bf16" else 4
    summ_bytes = (w.B * w.Hkv * w.Nc * w.S * w.d * el + 2 * w.B * w.Hq * w.Nc * w.d * el + 4 * w.B * w.Hq * w.Nc)
    out = torch.empty_like(x["q"])
    M = w.T
    lse = torch.empty((w.B, w.Hq) if M == 1 else (w.B, w.Hq, M), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.Hkv, w.topk) if M == 1 else (w.B, w.Hkv, M, w.topk), dtype=torch.int32, device=dev)
    p = H.make_params(w.B, M, w.L, w.Hq, w.Hkv, w.d, w.S, w.topk, w.W, w.L - M)
    ws = torch.empty(H.workspace_size(p, H.OP_DECODE), dtype=torch.uint8, device=dev)

    def one():
        H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk, window=w.W,
                 out=out, lse=lse, idx_out=idx, workspace=ws)

    # capture `steps` decode steps in one CUDA graph (the per-step footprint exceeds L2: no flush)
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        for _ in range(3):
            one()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            one()

    def run(mark):
        graph.replay()
        mark()

    _, total_ms, clocks = timed_steps(1, run, max(3, args.warmup // 3), None, dist,
                                      ClockSampler(physical_gpu_index(dist.local_rank)))
    needles_found = 0
    for b in range(w.B):
        first = idx[b, 0] if w.T == 1 else idx[b, 0, 0]  # the needle keys follow the first query's q^
        needles_found += len(set(x["needle_chunks"][b].tolist()) & set(first.tolist()))
    ms_step = dist.max(total_ms / steps)  # per-sequence-batch latency: the slowest rank's
    nbytes = decode_bytes(w, idx)
    gbs = nbytes["total"] / (ms_step / 1e3) / 1e9
    del graph
    summ = {"ms": summ_ms, "bytes": summ_bytes, "achieved_gbs": summ_bytes / (summ_ms / 1e3) / 1e9,
            "peak_gbs": peaks["hbm_gbs"], "frac": summ_bytes / (summ_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "note": "hils_chunk_summary over the whole cache: K and landmark queries read, k' and b' written"}
    return {"workload": w.name, "query_tokens_per_step": M, "us_per_step": ms_step * 1e3,
            "us_per_token": ms_step * 1e3 / M, "us_per_step_per_seq": ms_step * 1e3 / w.B,
            "summaries": summ,
            "steps": steps, "bytes_per_step": nbytes,
            "roofline": {"bound": "hbm", "kernel": "hils_decode (whole step: score, select, attend, combine)",
                         "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "traffic": None},
            "needle_recall": needles_found / max(1, w.B * min(w.needles, w.Nc)), "clocks": clocks,
            "launches_per_step": 4}


def bench_bsa(args, dist, dev, H, peaks):
    """Naive BSA selection (exact chunk masses over every pre-window token + the group top-k) at the
    prefill workload: the reference the HiLS selection approximates. Algorithmic flops: 2 d per (row,
    head, candidate token)."""
    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=rank_seed(1000, dist.rank), device=dev)
    idx = torch.empty((w.B, w.Hkv, w.T, w.topk), dtype=torch.int32, device=dev)
    mass = torch.empty((w.B, w.Hq, w.T, w.Nc), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(mark):
        H.bsa_select_topk(x["q"], x["k"], S=w.S, topk=w.topk, window=w.W, idx=idx, mass=mass)
        mark()

    steps = max(1, min(args.steps, 10))
    _, total_ms, _ = timed_steps(steps, step, 3, flush, dist)
    ms = dist.max(total_ms / steps)
    cand_tokens = sum(window_left(p, w.W, w.S) for p in range(w.T)) * w.B * w.Hq
    flops = 2 * w.d * cand_tokens
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": w.name, "ms": ms, "flops": flops,
            "roofline": {"bound": "tensor", "kernel": "hils_bsa_select_topk (masses + top-k)", "achieved": tf,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                         "traffic": None},
            "launches_per_step": 2}


def bench_select_qcal(args, dist, dev, H):
    """Selection with Q-Cal fused (q^ formed from q in shared memory) against the plain selection on a
    precomputed q^, both at the prefill workload on the same summaries."""
    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=rank_seed(1000, dist.rank), device=dev)
    k_sum, b_sum = H.chunk_summary(x["k"], x["q_land"], w.S)
    idx = torch.empty((w.B, w.Hkv, w.T, w.topk), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(mark):
        H.select_topk_qcal(x["q"], x["w_down"], x["w_up"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk,
                           window=w.W, idx=idx)
        mark()
        H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W, idx=idx)
        mark()

    steps = max(1, min(args.steps, 10))
    stage_ms, _, _ = timed_steps(steps, step, 3, flush, dist)
    return {"workload": w.name, "fused_ms": dist.max(stage_ms[0] / steps), "unfused_ms": dist.max(stage_ms[1] / steps),
            "note": "fused: hils_select_topk_qcal from q, W_down, W_up; unfused: hils_select_topk from q^"}


def bench_prefill_local(args, dist, dev, H, peaks):
    """The prefill attention on position-correlated queries (recipe "local": adjacent queries select
    overlapping chunks, the regime the query packing of Sec. 4 assumes), next to the union ratio of the
    selections: chunks a 32-query tile visits (window and selected) per chunk one query attends."""
    w = W.PREFILL_LOCAL_BF16
    x = W.prefill_inputs(w, seed=rank_seed(1000, dist.rank), device=dev)
    out, lse, idx, k_sum, b_sum = H.prefill(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], S=w.S, topk=w.topk,
                                            window=w.W)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    _, _, shat = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                               with_shat=True)

    def step(mark):
        H.attn_fwd_shat(x["q"], x["k"], x["v"], idx, shat, S=w.S, window=w.W, out=out, lse=lse)
        mark()

    steps = max(1, min(args.steps, 10))
    _, total_ms, _ = timed_steps(steps, step, 3, flush, dist)
    ms = dist.max(total_ms / steps)
    work = prefill_work(w)
    tf = work["attn_flops"] / (ms / 1e3) / 1e12
    return {"workload": w.name, "attn_ms": ms, "achieved_tflops": tf, "frac": tf / peaks["bf16_tflops"],
            **packing_stats(w, idx),
            "note": "hils_attn_fwd_shat alone on its own selection; algorithmic flops as in the headline"}


def packing_stats(w: W.Workload, idx) -> dict:
    """Selected chunks per query against distinct selected chunks per tile of 128 / G queries (the rows
    one attention CTA packs): how much of a tile's selected-chunk work each row actually uses."""
    QT = 128 // w.G
    nt = w.T // QT
    sel = idx[:, :, :nt * QT].reshape(w.B, w.Hkv, nt, QT * w.topk).long()
    hit = torch.zeros((w.B, w.Hkv, nt, w.Nc + 1), dtype=torch.bool, device=idx.device)
    hit.scatter_(3, torch.where(sel < 0, torch.full_like(sel, w.Nc), sel), True)
    return {"selected_chunks_per_query": (idx >= 0).sum(-1).double().mean().item(),
            "selected_chunks_per_tile": hit[..., :w.Nc].sum(-1).double().mean().item(),
            "queries_per_tile": QT}


def bench_train(args, dist, dev, H, peaks):
    w = W.TRAIN_BF16
    x = W.prefill_inputs(w, seed=rank_seed(3000, dist.rank), device=dev, with_dout=True)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(mark):
        out, lse, idx, k_sum, b_sum = H.prefill(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], S=w.S,
                                                topk=w.topk, window=w.W)
        mark()
        H.attn_bwd(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], k_sum, b_sum, idx, out, lse, x["dout"], S=w.S,
                   window=w.W)
        mark()

    steps = max(1, min(args.steps, 5))
    stage_ms, total_ms, _ = timed_steps(steps, step, 1, flush, dist)
    work = prefill_work(w)
    fwd_flops = work["attn_flops"] + work["route_flops"] + work["summary_flops"]
    bwd_flops = work["attn_flops"] * 14 // 4 + 2 * work["summary_flops"]
    ms, tps = weak_scaling_value(dist, total_ms / steps, w.B * w.T)
    return {"workload": w.name, "tokens_per_s": tps, "ms_per_step": ms,
            "fwd_ms": stage_ms[0] / steps, "bwd_ms": stage_ms[1] / steps,
            "roofline": {"bound": "tensor", "kernel": "hils_attn_bwd",
                         "achieved": bwd_flops / (stage_ms[1] / steps / 1e3) / 1e12,
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": bwd_flops / (stage_ms[1] / steps / 1e3) / 1e12 / peaks["bf16_tflops_sustained"],
                         "traffic": None, "note": "bwd flops = 14*d per (row, head, attended token) + summary bwd"},
            "launches_per_step": 5}


# ----------------------------------------------------------------------------- CPU (oracle)

def oracle_prefill_sample(x_cpu, w: W.Workload, groups, row_blocks, block_rows, budget_s=None):
    """The oracle on a bounded sample of the prefill workload: for each listed (b, KV group), all of
    its summaries, then selection + attention for up to `row_blocks` evenly spaced blocks of
    `block_rows` query rows (visited in a stratified order, stopping once `budget_s` seconds have
    passed). Returns (seconds, equivalent tokens = rows * G / Hq, blocks done)."""
    import oracle
    from oracle import Geometry

    def np64(t):
        return t.to(torch.float64).numpy()

    order = sorted(range(row_blocks), key=lambda r: int(format(r, "016b")[::-1], 2))  # bit-reversal strata
    rows_done, blocks_done = 0, 0
    t0 = time.perf_counter()
    for b, grp in groups:
        hs = slice(grp * w.G, (grp + 1) * w.G)
        kk = np64(x_cpu["k"][b:b + 1, grp:grp + 1])
        vv = np64(x_cpu["v"][b:b + 1, grp:grp + 1])
        g1 = Geometry(B=1, T=1, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W)
        ks, bs = oracle.chunk_summary(g1, kk, np64(x_cpu["q_land"][b:b + 1, hs]))
        for r in order:
            if budget_s is not None and blocks_done > 0 and time.perf_counter() - t0 > budget_s:
                break
            r0 = int((w.T - block_rows) * (r + 0.5) / row_blocks)
            gr = Geometry(B=1, T=block_rows, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=r0)
            rows = slice(r0, r0 + block_rows)
            qh = np64(x_cpu["q_hat"][b:b + 1, hs, rows])
            idx, _ = oracle.select_topk(gr, qh, ks, bs)
            oracle.attn_fwd(gr, np64(x_cpu["q"][b:b + 1, hs, rows]), kk, vv, qh, ks, bs, idx)
            rows_done += block_rows
            blocks_done += 1
    secs = time.perf_counter() - t0
    return secs, rows_done * w.G / w.Hq, blocks_done


ORACLE_BLOCKS, ORACLE_BLOCK_ROWS = 64, 128


def oracle_sample_text(w: W.Workload, slices: int) -> str:
    return (f"{slices} (batch, KV group) slice(s) of the prefill workload, each with all its {w.Nc} chunk summaries "
            f"and {ORACLE_BLOCKS} evenly spaced blocks of {ORACLE_BLOCK_ROWS} query rows (all {w.G} heads); "
            f"tokens counted as rows*G/Hq")


def cpu_baseline(x_gpu, w, budget_s=15.0):
    """The oracle as it stands on the host cores: whole (batch, KV group) slices (see oracle_sample_text)
    until about `budget_s` seconds of CPU time are spent."""
    import oracle

    x_cpu = {n: x_gpu[n].cpu() for n in ("q", "k", "v", "q_hat", "q_land")}
    groups = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    secs, tokens = 0.0, 0.0
    done = []
    for bg in groups:  # whole (batch, group) slices until the time budget is spent
        s, t, _ = oracle_prefill_sample(x_cpu, w, [bg], ORACLE_BLOCKS, ORACLE_BLOCK_ROWS)
        secs, tokens = secs + s, tokens + t
        done.append(bg)
        if secs > budget_s:
            break
    return {"value": tokens / secs, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": oracle_sample_text(w, len(done)) + f"; {secs:.1f} s of CPU time"}


def run_reference(args, dist):
    """Reference arm: the fp64 CPU oracle on the host cores, one step = the same sample unit as the
    cpu_baseline leg (one whole (batch, KV group) slice), the slices visited in turn. Under torchrun only
    rank 0 runs it; the other ranks exit without work."""
    if dist.rank != 0:
        return
    import oracle

    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=1000, device="cpu")
    groups = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    for n in range(args.warmup):
        oracle_prefill_sample(x, w, [groups[n % len(groups)]], ORACLE_BLOCKS, ORACLE_BLOCK_ROWS)
    total, tokens = 0.0, 0.0
    for n in range(args.steps):
        s, t, _ = oracle_prefill_sample(x, w, [groups[n % len(groups)]], ORACLE_BLOCKS, ORACLE_BLOCK_ROWS)
        total += s
        tokens += t
    value = tokens / total
    line = {"metric": METRIC, "value": value,
            "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": base_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": oracle_sample_text(w, 1) + " per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ----------------------------------------------------------------------------- profiling cases

def profile_case(args):
    """`--profile STAGE`: `args.steps` untimed launches of one stage on its workload, for ncu captures of
    one kernel (select it with ncu's -k / -s / -c). Prints no bench line. The summary case runs on a
    128K-token cache (B1; 256 MiB of keys, above L2), the decode case on a 512K-token cache at B1 (2 GiB of
    K and V: the decode workload's per-sequence shape with a footprint a profiler can save and restore)."""
    import chunk_wise_hierarchical_summary_b200.hils as H

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    st = args.profile
    if st in ("summary", "decode", "decode_multi"):
        w = W.decode_sweep(524288) if st != "summary" else W.decode_sweep(131072)
        if st == "decode_multi":
            w = w.with_(name="decode_m4_bf16_B1_L524288", T=4, q_pos0=w.L - 4)
        x = W.decode_inputs(w, seed=2000, device=dev)
        k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
        if st == "summary":
            fn = lambda: H.chunk_summary(x["k_cache"], x["q_land"], w.S, k_sum=k_sum, b_sum=b_sum)
        else:
            fn = lambda: H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                                  window=w.W)
    else:
        w = W.TRAIN_BF16 if st == "bwd" else W.PREFILL_BF16
        x = W.prefill_inputs(w, seed=1000, device=dev, with_dout=(st == "bwd"))
        out, lse, idx, k_sum, b_sum = H.prefill(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], S=w.S, topk=w.topk,
                                                window=w.W)
        if st == "select":
            fn = lambda: H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                       idx=idx)
        elif st == "select_qcal":
            fn = lambda: H.select_topk_qcal(x["q"], x["w_down"], x["w_up"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S,
                                            topk=w.topk, window=w.W, idx=idx)
        elif st == "bsa":
            mass = torch.empty((w.B, w.Hq, w.T, w.Nc), dtype=torch.float32, device=dev)
            fn = lambda: H.bsa_select_topk(x["q"], x["k"], S=w.S, topk=w.topk, window=w.W, idx=idx, mass=mass)
        elif st == "attn":
            _, _, shat = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                       with_shat=True)
            fn = lambda: H.attn_fwd_shat(x["q"], x["k"], x["v"], idx, shat, S=w.S, window=w.W, out=out, lse=lse)
        elif st == "attn_gather":
            fn = lambda: H.attn_fwd(x["q"], x["k"], x["v"], x["q_hat"], k_sum, b_sum, idx, S=w.S, window=w.W,
                                    out=out, lse=lse)
        else:
            fn = lambda: H.attn_bwd(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], k_sum, b_sum, idx, out, lse,
                                    x["dout"], S=w.S, window=w.W)
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    H.check()
    print(f"profile case {st} on {w.name}: {args.steps} launches done")


# ----------------------------------------------------------------------------- main

def decode_summary(decode: dict, extra: dict) -> dict:
    """The decode half of the headline in a few fields: us/token and the HBM fraction at the decode
    workload, then the sweep's (L, us/token, HBM fraction) and multi-token decode, when run."""
    out = {"workload": decode["workload"], "us_per_token": decode["us_per_token"],
           "hbm_frac": decode["roofline"]["frac"], "achieved_gbs": decode["roofline"]["achieved"],
           "peak_gbs": decode["roofline"]["peak"], "bytes_per_step": decode["bytes_per_step"]["total"],
           "l2": "not flushed: one fixed query per sequence replayed, 629 MB touched per step (5x L2)"}
    if "decode_sweep" in extra:
        out["sweep_L_us_frac"] = [[r["L"], round(r["us_per_token"], 2), round(r["hbm_frac"], 4)]
                                  for r in extra["decode_sweep"]]
    if "decode_multi" in extra:
        m = extra["decode_multi"]
        out["multi_m4_us_per_step"] = m["us_per_step"]
        out["multi_m4_hbm_frac"] = m["roofline"]["frac"]
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hils", choices=("hils", "reference"))
    ap.add_argument("--quick", action="store_true", help="headline only (no decode sweep / training blocks)")
    ap.add_argument("--profile",
                    choices=("summary", "select", "select_qcal", "attn", "attn_gather", "decode", "decode_multi", "bwd",
                             "bsa"),
                    help="run --steps untimed launches of one stage for an ncu capture; no bench line")
    args = ap.parse_args()
    if args.profile:
        profile_case(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, dist)
            return
        import chunk_wise_hierarchical_summary_b200.hils as H

        dev = torch.device("cuda", dist.local_rank)
        torch.cuda.set_device(dev)
        peaks, peak_src = load_peaks()
        pre = bench_prefill(args, dist, dev, H, peaks)
        w = pre["workload"]
        ms, value = weak_scaling_value(dist, pre["ms_per_step"], w.B * w.T)
        e2e = bench_prefill_e2e(args, dist, dev, H, pre)
        decode = bench_decode(args, dist, dev, H, peaks, W.DECODE_BF16, 256)
        extra = {}
        if not args.quick:
            extra["decode_sweep"] = []
            for L in W.DECODE_SWEEP_L:
                r = bench_decode(args, dist, dev, H, peaks, W.decode_sweep(L), 64)
                extra["decode_sweep"].append({"L": L, "us_per_token": r["us_per_token"],
                                              "bytes_per_step": r["bytes_per_step"]["total"],
                                              "hbm_frac": r["roofline"]["frac"], "needle_recall": r["needle_recall"]})
            # multi-token decode (M = 4 query tokens per sequence and step, e.g. speculative verification)
            wm = W.DECODE_BF16.with_(name="decode_m4_bf16_B8_L524288_Hq32_Hkv8_d128_S64_k32_W512", T=4,
                                     q_pos0=W.DECODE_BF16.L - 4)
            extra["decode_multi"] = bench_decode(args, dist, dev, H, peaks, wm, 64)
            extra["train"] = bench_train(args, dist, dev, H, peaks)
            extra["bsa_select"] = bench_bsa(args, dist, dev, H, peaks)
            extra["select_qcal"] = bench_select_qcal(args, dist, dev, H)
            extra["prefill_local"] = bench_prefill_local(args, dist, dev, H, peaks)
        cpu = None
        if dist.world == 1:
            cpu = cpu_baseline(pre["x"], w)
        launches = pre["launches_per_step"] * args.steps
        pre["roofline"]["peak_source"] = peak_src
        line = {
            "metric": METRIC,
            "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": base_config(w, dist.world),
            "stage_ms": {"chunk_summary": pre["stage_ms"][0], "select_topk": pre["stage_ms"][1],
                         "attn_fwd_shat": pre["stage_ms"][2]},
            "roofline": pre["roofline"],
            "packing": packing_stats(w, pre["idx"]),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": pre["clocks"],
            **extra,
            "decode_detail": decode,
            # last, so that the headline's decode half is in any tail of the line
            "decode": decode_summary(decode, extra),
        }
        if dist.rank == 0:
            print(json.dumps(line, default=lambda o: getattr(o, "name", str(o))))
    finally:
        dist.close()


if __name__ == "__main__":
    main()
