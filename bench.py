"""Benchmark of the block-sparse paged attention hot path on B200.

One step = one pass of the whole path over one batch: block scores -> selection -> sparse
paged attention (split-K + combine), through the C ABI.  The headline workload is the largest
single-GPU configuration, FP8 long-context decode (batch 128, 1 query token, 8 KV heads x 8
query heads, head dim 128, context 131072, e4m3 KV, BF16 index-K, page 128, top_k 64, init 1,
local 4: 6.6 GB of algorithmic HBM traffic per step); the four other workloads are measured
the same way in the same run and reported under "workloads".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--only]
                    [--impl ours|reference]

Timing: W warm-up steps, then blocks of exactly K steps (CUDA events on the launching stream,
synchronize and barrier on both sides) repeated for about a second; the median block gives
the value.  Per-launch times come from separate passes with events between the launch groups.
Under torchrun every rank runs an independent replica (the path does not shard: no
collective), and rank 0 prints one JSON line whose value is the query tokens of all ranks
divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "sparse-attn query-tokens/s and achieved HBM GB/s (% of roofline) at 1 B200"
UNIT = "query-tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    ws, rank, _ = dist_env()
    if ws > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))
    return ws, rank


def barrier(ws: int, device=None):
    if ws > 1:
        if device is not None and torch.distributed.get_backend() == "nccl":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(x: float, ws: int, device) -> float:
    """The largest value of x over all ranks (every rank calls it, in the same order)."""
    if ws == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ peaks and clocks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) while the timed region runs."""
    QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.rows, self.proc, self.thread = index, [], None, None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [r for (t, r) in self.rows if t0 - 0.15 <= t <= t1 + 0.15] or \
            [r for (_, r) in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx.append(float(r[1]))
            except ValueError:
                continue
            for n, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


# ------------------------------------------------------------------ algorithmic work
# index-K bytes per token and head: bf16; e4m3 + f32 scale; e2m1 pairs + 4 UE8M0 exponents
INDEX_K_TOKEN_BYTES = {"bf16": 256, "fp8": 132, "fp4": 68}


def algorithmic_bytes(prob, block_ids, num_selected, shared=False):
    """HBM bytes the method itself must move per step (implementation traffic excluded):
    index: every visible index-K position of every sequence (only the first new token's, with
    the top-k shared across draft tokens) (+ q_idx); attention: K and V of every valid
    position of each (sequence, KV head)'s union of selected blocks (+ q, out)."""
    import numpy as np
    BLOCK, D = 128, 128
    kv_elem = 1 if prob["kv_fp8"] else 2
    ro = prob["row_off"].cpu().tolist()
    cl = prob["cache_len"].cpu().tolist()
    L = prob["kv_lens"]
    ids = block_ids.cpu().numpy()
    cnt = num_selected.cpu().numpy()
    tok_bytes = INDEX_K_TOKEN_BYTES[prob.get("idx_dtype", "bf16")]
    seen = [(cl[b] + 1 if shared else L[b]) for b in range(prob["batch"]) if ro[b + 1] > ro[b]]
    idx_bytes = sum(seen) * prob["H_idxk"] * tok_bytes + \
        (prob["batch"] if shared else prob["total_q"]) * prob["H_kv"] * D * 2
    kv_bytes = 0
    for b in range(prob["batch"]):
        if ro[b + 1] == ro[b]:
            continue
        for g in range(prob["H_kv"]):
            blocks = set()
            for t in range(ro[b], ro[b + 1]):
                blocks.update(ids[t, g, :cnt[t, g]].tolist())
            for j in blocks:
                kv_bytes += min(BLOCK, L[b] - j * BLOCK) * D * kv_elem * 2
    qo_bytes = prob["total_q"] * prob["H_q"] * D * 2 * 2
    return idx_bytes, kv_bytes + qo_bytes


def algorithmic_flops(prob, block_ids, num_selected):
    """FLOPs the method itself needs per step (masked work a tiled kernel executes is not
    counted): index stage 2*128*(p+1) per (token, index-query head); attention
    4*128*|P(t,g)| per (token, query head) with P(t,g) the selected, causally clipped
    positions."""
    import numpy as np
    BLOCK, D = 128, 128
    ro = prob["row_off"].cpu().numpy()
    cl = prob["cache_len"].cpu().numpy()
    q_lens = np.diff(ro)
    b_of_t = np.repeat(np.arange(prob["batch"]), q_lens)
    p = cl[b_of_t] + (np.arange(prob["total_q"]) - ro[b_of_t])           # [tq]
    idx_flops = float((2 * D * (p + 1)).sum()) * prob["H_kv"]
    ids = block_ids.cpu().numpy().astype(np.int64)                         # [tq, H_kv, S]
    cnt = num_selected.cpu().numpy()
    valid = np.arange(ids.shape[2])[None, None, :] < cnt[:, :, None]
    cover = np.clip(p[:, None, None] + 1 - ids * BLOCK, 0, BLOCK)
    positions = np.where(valid, cover, 0).sum(axis=2)                      # [tq, H_kv]
    G = prob["H_q"] // prob["H_kv"]
    attn_flops = float(positions.sum()) * G * 4 * D
    return idx_flops, attn_flops


def executed_flops_tiles(prob, block_ids, num_selected, tile_tokens):
    """FLOPs a tile-union kernel executes: per (query tile, KV head) every block of the
    union of its tokens' selections, on full 128-row x 128-position x 128-dim tiles
    (QK^T and PV)."""
    import numpy as np
    ro = prob["row_off"].cpu().numpy()
    ids = block_ids.cpu().numpy()
    cnt = num_selected.cpu().numpy()
    blocks = 0
    for b in range(prob["batch"]):
        for t0 in range(ro[b], ro[b + 1], tile_tokens):
            t1 = min(t0 + tile_tokens, ro[b + 1])
            for g in range(prob["H_kv"]):
                sel = [ids[t, g, :cnt[t, g]] for t in range(t0, t1)]
                blocks += len(np.unique(np.concatenate(sel))) if sel else 0
    return float(blocks) * 4 * 128 * 128 * 128


def source_digest(*names):
    """Digest of a kernel's code: its source file and the headers that hold its math, with
    comments and all white space removed (a comment or layout edit does not make a profile
    stale)."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "block_sparse_paged_scores_b200", "csrc", n)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, digest: str):
    """DRAM bytes per launch from a committed ncu summary, when it was taken on this exact
    kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        e = d[f"{kernel}/{workload}"]
        return float(e["dram_bytes_per_launch"]) if e.get("source_digest") == digest else None
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(workload: str, n_seq: int, seed: int):
    """A bounded sample of a workload (or of a variant: its workload with the variant's
    changes) for the CPU oracle, its description, and whether the indexer top-k is shared
    across draft tokens.  Decode-like workloads: n_seq of their sequences (same
    distributions).  Prefill: one sequence with 16-64 new tokens over a prior cache drawn as in
    the workload (a whole prefill sequence is minutes of fp64 work per pass)."""
    from block_sparse_paged_scores_b200 import workload as wl
    base, changes, path_kw = VARIANTS.get(workload, (workload, {}, {}))
    spec = wl.WORKLOADS[base].scaled(**changes)
    share = bool(path_kw.get("share_selection"))
    q_hi = spec.q_len[1] if isinstance(spec.q_len, tuple) else spec.q_len
    if q_hi > 8:
        p = wl.generate(spec.scaled(batch=1, q_len=(16, 64)), seed=seed)
        desc = (f"1 of {spec.batch} sequences of {workload} with {p['total_q']} new tokens "
                f"(16-64 instead of the workload's q_len; prior cache as in the workload)")
    else:
        p = wl.generate(spec.scaled(batch=min(n_seq, spec.batch)), seed=seed)
        desc = f"{p['batch']} of {spec.batch} sequences of {workload} (same distributions)"
    return p, desc, share


def time_oracle(prob, min_seconds: float, max_seconds: float, share: bool = False):
    import oracle
    oracle.build()
    tokens, t0, reps = 0, time.perf_counter(), 0
    while True:
        oracle.forward(prob, prob["top_k"], prob["init_blocks"], prob["local_blocks"],
                       prob["scale"], prob["max_blocks"], share=share)
        tokens += prob["total_q"]
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el * (reps + 1) / reps > max_seconds:
            return tokens / el, el, reps


def cpu_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ timing helpers
def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def blocks_for(block_ms: float, min_s: float, ws: int, dev) -> int:
    """How many K-step blocks fill about ``min_s`` seconds (at least 3): the same count on every
    rank (the largest over ranks), so that every rank takes the same steps."""
    n = max(3, min(2000, math.ceil(min_s * 1e3 / max(block_ms, 1e-3))))
    return int(max_over_ranks(n, ws, dev))


def time_block(step, steps: int, stream, flush_buf=None) -> float:
    """Device time (ms) of one block of ``steps`` calls of step() on ``stream``, from CUDA
    events on that stream with a synchronize on both sides.  With ``flush_buf`` L2 is flushed
    before every step (a write of twice its size, outside the step's own events) and the
    steps' own intervals are summed."""
    torch.cuda.synchronize()
    if flush_buf is None:
        e0, e1 = _events(2)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)
    evs = [_events(2) for _ in range(steps)]
    for a_, b_ in evs:
        flush_buf.fill_(1)
        a_.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    return sum(a_.elapsed_time(b_) for a_, b_ in evs)


def stage_times(groups, steps: int, stream, min_s: float):
    """Each launch group's average device time per step (ms): K-step passes with an event
    between consecutive groups, repeated until about ``min_s`` seconds have passed (at least
    three passes); the median over the passes."""
    per = [[] for _ in groups]
    t0 = time.perf_counter()
    while True:
        evs = [_events(len(groups) + 1) for _ in range(steps)]
        for k in range(steps):
            evs[k][0].record(stream)
            for i, fn in enumerate(groups):
                fn()
                evs[k][i + 1].record(stream)
        torch.cuda.synchronize()
        for i in range(len(groups)):
            per[i].append(sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps))
                          / steps)
        if len(per[0]) >= 3 and time.perf_counter() - t0 >= min_s:
            return [statistics.median(x) for x in per]


# ------------------------------------------------------------------ arms
def run_reference(args):
    """The CPU oracle as the reference arm: each step is the whole path on a bounded sample
    of the workload (a few of its sequences, same distributions)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    prob, desc, share = oracle_sample(args.workload, args.cpu_sample_seqs, seed=7)
    import oracle
    oracle.build()
    fwd = lambda: oracle.forward(prob, prob["top_k"], prob["init_blocks"], prob["local_blocks"],
                                 prob["scale"], prob["max_blocks"], share=share)
    for _ in range(args.warmup):
        fwd()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fwd()
    el = time.perf_counter() - t0
    value = prob["total_q"] * args.steps / el
    cores = cpu_threads()
    sample = f"{desc}, seed 7, per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# Variants of the five workloads with the options the pages add: the index-K cache in a scaled
# format (TensorRT-LLM DeepSeekSparseAttentionConfig, indexer_k_dtype) and the indexer top-k
# shared across draft tokens (index_share_for_mtp_iteration).  name -> (workload, spec
# changes, Path options)
VARIANTS = {
    "fp8_long_decode_fp8_index_k": ("fp8_long_decode", dict(idx_dtype="fp8"), {}),
    "fp8_long_decode_fp4_index_k": ("fp8_long_decode", dict(idx_dtype="fp4"), {}),
    "spec_decode_shared_topk": ("spec_decode", {}, dict(share_selection=True)),
    # ragged prefill whose index queries are coherent across neighbouring tokens (a 256-token
    # moving average of N(0,1) draws, neighbour correlation about 0.996): the tokens of a tile
    # select similar blocks, as the queries of a trained model do, instead of independent
    # random sets
    "ragged_prefill_coherent_queries": ("ragged_prefill", dict(q_idx_window=256), {}),
    # ragged prefill over a scale-free FP8 e4m3 KV cache (the tcgen05 kernel converts the tiles
    # to f16 in shared memory)
    "ragged_prefill_fp8_kv": ("ragged_prefill", dict(kv_dtype="fp8"), {}),
}


def bench_workload(name, args, ws, rank, dev, sampler, with_cpu):
    """Every measurement of one workload: the timed whole-path step (median of repeated
    K-step blocks), per-launch times of the same launches, the roofline of the dominant one,
    the end-to-end figure with host buffers and, when asked, the CPU oracle baseline."""
    from block_sparse_paged_scores_b200 import msa
    from block_sparse_paged_scores_b200 import workload as wl

    base, changes, path_kw = VARIANTS.get(name, (name, {}, {}))
    spec = wl.WORKLOADS[base].scaled(**changes)
    if args.batch:
        spec = spec.scaled(batch=args.batch)
    prob = wl.generate(spec, seed=wl.SEEDS[base] + 1000 * rank, device=dev)
    path = msa.Path(prob, num_splits=args.splits, **path_kw)
    shared = bool(path_kw.get("share_selection"))
    stream = torch.cuda.current_stream(dev)
    fp8 = prob["kv_fp8"]
    G = prob["H_q"] // prob["H_kv"]
    decode = prob["max_q_len"] == 1 and G <= 16      # the selection runs inside the attention
    stream_route = prob["max_q_len"] <= 8            # persistent split-K kernel (+ combine)
    tensor_route = not stream_route                  # prefill: dense contractions, tcgen05
    splits = msa.msa_attn_partials(path.rp, prob["S"], prob["H_q"], prob["H_kv"],
                                   path.max_blocks, args.splits)[0] if stream_route else 1
    combine = stream_route and splits > 1
    if shared:          # index with the selection inside, plan, attention, [combine]
        launches = 3 + int(combine)
    elif decode:        # index, attention with the selection inside, [combine]
        launches = 2 + int(combine)
    elif stream_route:  # index, select, plan, attention, [combine]
        launches = 4 + int(combine)
    else:               # index, select, plan, attention
        launches = 4
    step = lambda: path.run(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert int(path.dev_err.item()) == 0, f"device error flag set during warm-up ({name})"

    idx_bytes, attn_bytes = algorithmic_bytes(prob, path.block_ids, path.num_selected, shared)
    flush = idx_bytes + attn_bytes < L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None

    # ---- the timed region: blocks of exactly K steps between barriers, repeated for about
    # args.min_seconds; the median block is the number
    first = time_block(step, args.steps, stream, flush_buf)
    n_blocks = blocks_for(first, args.min_seconds, ws, dev)
    barrier(ws, dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    blocks = [time_block(step, args.steps, stream, flush_buf) for _ in range(n_blocks)]
    barrier(ws, dev)
    t_wall1 = time.time()
    ms_block = max_over_ranks(statistics.median(blocks), ws, dev)
    tokens = sum_over_ranks(prob["total_q"], ws, dev)
    assert int(path.dev_err.item()) == 0, f"device error flag set ({name})"

    # ---- the same launches, one group at a time (events between them)
    if shared:
        groups = {"index_select_shared": lambda: path.index_select(stream)}
        attn_key = "attention_incl_plan"
        if combine:
            groups[attn_key] = lambda: path.attend(stream=stream, combine=False)
            groups["combine"] = lambda: path.combine(stream)
        else:
            groups[attn_key] = lambda: path.attend(stream=stream)
        attn_src = ("attention_stream.cu", "attn_common.cuh", "select_row.cuh")
    elif decode:
        groups = {"index_scores": lambda: path.index_scores(stream)}
        if combine:
            groups["attention_with_selection"] = lambda: path.select_attend(stream,
                                                                            combine=False)
            groups["combine"] = lambda: path.combine(stream)
        else:
            groups["attention_with_selection"] = lambda: path.select_attend(stream)
        attn_key = "attention_with_selection"
        attn_src = ("attention_stream.cu", "attn_common.cuh", "select_row.cuh")
    else:
        groups = {"index_scores": lambda: path.index_scores(stream),
                  "select": lambda: path.select(stream=stream)}
        attn_key = "attention_incl_plan"
        if combine:
            groups[attn_key] = lambda: path.attend(stream=stream, combine=False)
            groups["combine"] = lambda: path.combine(stream)
        else:
            groups[attn_key] = lambda: path.attend(stream=stream)
        attn_src = (("attention_stream.cu", "attn_common.cuh", "select_row.cuh")
                    if stream_route else ("attention_tc.cu",))
    idx_src = (("indexer.cu", "select_row.cuh")
               if stream_route or prob["idx_dtype"] != "bf16" else ("indexer_tc.cu",))
    st = stage_times(list(groups.values()), args.steps, stream, args.stage_seconds)
    stages = dict(zip(groups, st))
    if stream_route and not shared:
        # for comparison: the first two stages as one msa_index_select launch
        stages["fused_index_select"] = stage_times([lambda: path.index_select(stream)],
                                                   args.steps, stream,
                                                   args.stage_seconds / 2)[0]

    # ---- roofline of the dominant launch group of the step
    hbm, bf16, bf16_sus, peak_src = measured_peaks()
    idx_key = "index_select_shared" if shared else "index_scores"
    kinds = {idx_key: (stages[idx_key], idx_src), attn_key: (stages[attn_key], attn_src)}
    dom = max(kinds, key=lambda k: kinds[k][0])
    d_ms, d_src = kinds[dom]
    traffic_kernel = "index_scores" if dom == idx_key else "attention"
    traffic = profiled_traffic(traffic_kernel, name, source_digest(*d_src))
    if tensor_route:
        idx_flops, attn_flops = algorithmic_flops(prob, path.block_ids, path.num_selected)
        d_flops = idx_flops if dom == idx_key else attn_flops
        achieved = d_flops / (d_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": bf16,
                    "unit": "TFLOP/s", "frac": achieved / bf16, "peak_source": peak_src,
                    "frac_of_sustained_peak": achieved / bf16_sus, "traffic": traffic,
                    "algorithmic_flops_per_launch": d_flops,
                    "note": "algorithmic FLOPs (selected, causally clipped positions only) over "
                            "the launch group's median time, against the measured bf16 burst "
                            "peak"}
        if dom != idx_key:
            ex = executed_flops_tiles(prob, path.block_ids, path.num_selected, 128 // G)
            roofline["executed_flops_per_launch"] = ex
            roofline["executed_tflops"] = ex / (d_ms * 1e-3) / 1e12
            roofline["executed_frac"] = ex / (d_ms * 1e-3) / 1e12 / bf16
        work = {"algorithmic_tflop": (idx_flops + attn_flops) / 1e12,
                "achieved_TFLOPs": (idx_flops + attn_flops) / (ms_block / args.steps * 1e-3)
                / 1e12}
    else:
        d_bytes = idx_bytes if dom == idx_key else attn_bytes
        achieved = d_bytes / (d_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                    "unit": "GB/s", "frac": achieved / hbm, "peak_source": peak_src,
                    "frac_of_8TBps": achieved / 8000.0, "traffic": traffic,
                    "algorithmic_bytes_per_launch": d_bytes}
        step_s = ms_block / args.steps * 1e-3
        work = {"algorithmic_bytes": idx_bytes + attn_bytes,
                "achieved_GBps": (idx_bytes + attn_bytes) / step_s / 1e9,
                "frac_of_measured": (idx_bytes + attn_bytes) / step_s / 1e9 / hbm,
                "frac_of_8TBps": (idx_bytes + attn_bytes) / step_s / 8e12}

    # ---- end to end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and its output back, both inside the timed region
    e2e = None
    if not args.no_e2e:
        host = {k: prob[k].cpu().pin_memory() for k in msa.HostPipeline.PER_STEP}
        outs = [torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory()
                for _ in range(2)]
        d2h = outs[0].numel() * outs[0].element_size()

        def serial_step():
            for k_, v_ in host.items():
                prob[k_].copy_(v_, non_blocking=True)
            path.run(stream)
            outs[0].copy_(path.out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            serial_step()
        serial_ms = statistics.median(time_block(serial_step, args.steps, stream)
                                      for _ in range(3))
        pipe = msa.HostPipeline(prob, num_splits=args.splits, **path_kw)
        packed = pipe.pack(host)  # the step's inputs as one pinned buffer: one copy per step
        for i in range(max(2, args.warmup)):
            pipe.submit(packed, outs[i % 2])
        pipe.finish(stream)
        torch.cuda.synchronize(dev)

        def pipe_block():
            x0, x1 = _events(2)
            x0.record(stream)
            pipe.start(after=x0)
            for i in range(args.steps):
                pipe.submit(packed, outs[i % 2])
            pipe.finish(stream)
            x1.record(stream)
            torch.cuda.synchronize(dev)
            return x0.elapsed_time(x1)

        pipe_ms = statistics.median(pipe_block() for _ in range(3))
        for p_ in pipe.paths:
            assert int(p_.dev_err.item()) == 0, "device error flag set (host pipeline)"
        assert torch.equal(outs[(args.steps - 1) % 2].to(dev), path.out), \
            "host pipeline output differs from the device-resident step"
        pipe_ms = max_over_ranks(pipe_ms, ws, dev)
        serial_ms = max_over_ranks(serial_ms, ws, dev)
        e2e = {"value": tokens * args.steps / (pipe_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": packed.numel(), "d2h_bytes_per_step": d2h,
               "serial_value": tokens * args.steps / (serial_ms * 1e-3),
               "note": "per-step inputs (q, q_idx, row offsets, cache lengths, page table) "
                       "copied from pinned host memory and the output read back, every step "
                       "inside the timed region (median of 3 K-step blocks); value: two-deep "
                       "pipeline (the step's inputs packed in one pinned buffer, one copy; "
                       "step i+1's copy in and step i-1's copy out on their own streams while "
                       "step i computes); serial_value: one copy per input, compute, copy "
                       "out, all on one stream; the caches stay resident"}
        del pipe

    cpu = None
    if with_cpu:
        sample, desc, share = oracle_sample(name, args.cpu_sample_seqs, seed=7)
        v, el, reps = time_oracle(sample, args.cpu_min_s, args.cpu_max_s, share)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{desc}, seed 7, {reps} pass(es), {el:.1f} s"}

    l2 = ((f"{(idx_bytes + attn_bytes) / 2**20:.1f} MiB touched per step, under the "
           f"{L2_BYTES / 2**20:.0f} MiB L2: L2 flushed before every step (a "
           f"{2 * L2_BYTES / 2**20:.0f} MiB write outside the step's events), time = sum of "
           f"the steps' own intervals") if flush else
          (f"inputs larger than L2: {(idx_bytes + attn_bytes) / 2**20:.0f} MiB touched per "
           f"step vs {L2_BYTES / 2**20:.0f} MiB L2, no flush"))
    res = {
        "value": tokens * args.steps / (ms_block * 1e-3),
        "ms_per_step": ms_block / args.steps,
        "dtype": "fp8-e4m3 kv / bf16" if fp8 else "bf16",
        "config": {"workload": name, "batch": prob["batch"],
                   "q_tokens_per_step": prob["total_q"], "H_kv": prob["H_kv"],
                   "H_q": prob["H_q"], "head_dim": 128, "page_size": 128,
                   "top_k": prob["top_k"], "init_blocks": prob["init_blocks"],
                   "local_blocks": prob["local_blocks"],
                   "kv_lens": f"{spec.kv_len}" if spec.prior_len is None else
                   f"prior {spec.prior_len} + new {spec.q_len}",
                   "kv_dtype": spec.kv_dtype, "index_k_dtype": spec.idx_dtype,
                   "topk_shared_across_drafts": shared,
                   "split_k_partials": splits, "parallelism": f"replicas x{ws}", "l2": l2},
        "timing": {"blocks": n_blocks, "steps_per_block": args.steps,
                   "block_ms_min_median_max": [min(blocks), statistics.median(blocks),
                                               max(blocks)],
                   "note": "value and ms_per_step from the median block (max over ranks)"},
        "roofline": roofline,
        ("step_flops" if tensor_route else "step_hbm"): work,
        "stages_ms": stages,
        "launches_per_step": launches,
        "gpu_launches": launches * args.steps * n_blocks,
        "clocks": sampler.summary(t_wall0, t_wall1) if sampler else None,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    del path, prob, flush_buf
    torch.cuda.empty_cache()
    return res


def bench_latent(name, args, ws, rank, dev, sampler):
    """The latent sparse attention op (Mojo Struct_latent_sparse_attention_ragged_paged) on
    its decode workload: batch 64, 64 heads, a 128-position window, 512 compressed entries per
    query; measured like the other workloads (median of repeated K-step blocks)."""
    from block_sparse_paged_scores_b200 import msa
    from block_sparse_paged_scores_b200 import workload as wl

    spec = wl.LATENT_DECODE
    if args.batch:
        spec = spec.scaled(batch=args.batch)
    prob = wl.generate_latent(spec, seed=11 + 1000 * rank, device=dev)
    path = msa.LatentPath(prob)
    stream = torch.cuda.current_stream(dev)
    step = lambda: path.run(stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert int(path.dev_err.item()) == 0, "device error flag set (latent)"
    # algorithmic bytes: every latent row a query reads, once per query (K = V), + q and out
    ci = prob["comp_idx"].cpu()
    comp_len = prob["comp_len"].cpu()
    ro = prob["row_off"].cpu().tolist()
    rows = 0
    for b in range(prob["batch"]):
        for i in range(ro[b + 1] - ro[b]):
            p_ = int(prob["swa_len"][b]) + i
            rows += p_ - max(0, p_ - prob["window"] + 1) + 1
            e = ci[ro[b] + i]
            rows += int(((e >= 0) & (e < comp_len[b])).sum())
    alg_bytes = rows * 256 + prob["total_q"] * prob["H"] * 256 * 2
    flush = alg_bytes < L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    first = time_block(step, args.steps, stream, flush_buf)
    n_blocks = blocks_for(first, args.min_seconds, ws, dev)
    barrier(ws, dev)
    t_wall0 = time.time()
    blocks = [time_block(step, args.steps, stream, flush_buf) for _ in range(n_blocks)]
    barrier(ws, dev)
    t_wall1 = time.time()
    ms_block = max_over_ranks(statistics.median(blocks), ws, dev)
    tokens = sum_over_ranks(prob["total_q"], ws, dev)
    hbm, _, _, peak_src = measured_peaks()
    step_ms = ms_block / args.steps
    achieved = alg_bytes / (step_ms * 1e-3) / 1e9
    launches = 1 + int(path.num_splits > 1)
    res = {
        "value": tokens * args.steps / (ms_block * 1e-3), "ms_per_step": step_ms, "dtype": "bf16",
        "config": {"workload": name, "batch": prob["batch"], "q_tokens_per_step": prob["total_q"],
                   "heads": prob["H"], "latent_dim": 128, "window": prob["window"],
                   "compressed_entries_per_query": prob["n_entries"],
                   "splits": path.num_splits, "parallelism": f"replicas x{ws}",
                   "l2": (f"{alg_bytes / 2**20:.1f} MiB touched per step: L2 flushed before "
                          f"every step, time = sum of the steps' own intervals") if flush else
                         "inputs larger than L2, no flush"},
        "timing": {"blocks": n_blocks, "steps_per_block": args.steps,
                   "block_ms_min_median_max": [min(blocks), statistics.median(blocks),
                                               max(blocks)]},
        "roofline": {"bound": "hbm", "kernel": "latent_attention (+ combine)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "note": "a few MiB per step: bound by latency, not by HBM bandwidth"},
        "launches_per_step": launches, "gpu_launches": launches * args.steps * n_blocks,
        "clocks": sampler.summary(t_wall0, t_wall1) if sampler else None, "e2e": None,
    }
    del path, prob, flush_buf
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    from block_sparse_paged_scores_b200 import build as msa_build
    from block_sparse_paged_scores_b200 import msa
    from block_sparse_paged_scores_b200 import workload as wl

    ws, rank = init_dist("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        msa_build.build()
    barrier(ws, dev)
    msa.load()

    sampler = ClockSampler(local).start() if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    head = bench_workload(args.workload, args, ws, rank, dev, sampler,
                          with_cpu=rank == 0 and ws == 1 and not args.no_cpu_baseline)
    others = {}
    if not args.only:
        # the other workloads and the variants, each measured the same way (every rank takes
        # the same steps)
        for name in list(wl.WORKLOADS) + list(VARIANTS):
            if name != args.workload:
                others[name] = bench_workload(name, args, ws, rank, dev, sampler, False)
        others["latent_decode"] = bench_latent("latent_decode", args, ws, rank, dev, sampler)
    if sampler:
        sampler.stop()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic"}
    line.update({k: v for k, v in head.items() if k not in ("value", "ms_per_step", "dtype")})
    if others:
        line["workloads"] = {
            n: {k: r[k] for k in ("value", "ms_per_step", "dtype", "config", "timing",
                                  "roofline", "step_hbm", "step_flops", "stages_ms",
                                  "launches_per_step", "clocks", "e2e") if k in r}
            for n, r in others.items()}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fp8_long_decode",
                    help="the headline workload (the largest single-GPU configuration), or "
                    "another workload or variant to measure on its own (with --only)")
    ap.add_argument("--only", action="store_true",
                    help="measure the headline workload only (not the other four)")
    ap.add_argument("--splits", type=int, default=0, help="split-K partitions (0 = heuristic)")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="repeat K-step blocks for about this long; the median block counts")
    ap.add_argument("--stage-seconds", type=float, default=0.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--batch", type=int, default=0, help="override the workloads' batch "
                    "(profiling runs on a smaller case; not a bench number)")
    ap.add_argument("--cpu-sample-seqs", type=int, default=4)
    ap.add_argument("--cpu-min-s", type=float, default=10.0)
    ap.add_argument("--cpu-max-s", type=float, default=30.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from block_sparse_paged_scores_b200 import workload as wl
    if args.workload not in list(wl.WORKLOADS) + list(VARIANTS):
        ap.error(f"--workload: one of {', '.join(list(wl.WORKLOADS) + list(VARIANTS))}")
    if args.impl == "reference":
        return run_reference(args)
    rc = run_ours(args)
    ws, _, _ = dist_env()
    if ws > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
