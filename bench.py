"""Benchmark of the block-sparse paged attention hot path on B200.

One step = one pass of the whole path over one batch: block scores -> selection -> sparse
paged attention (split-K + combine), through the C ABI, on the BF16-decode workload (batch 32,
1 query token, 8 KV heads x 8 query heads, head dim 128, context U[16384, 65536], page 128,
top_k 16, init 1, local 2) unless --workload says otherwise.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun every rank runs an independent replica (the path does not shard: no
collective), timed on the device between barriers, and rank 0 prints one JSON line whose
value is the query tokens of all ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
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
def algorithmic_bytes(prob, block_ids, num_selected):
    """HBM bytes the method itself must move per step (implementation traffic excluded):
    index: every visible index-K position of every sequence (+ q_idx); attention: K and V of
    every valid position of each (sequence, KV head)'s union of selected blocks (+ q, out)."""
    import numpy as np
    BLOCK, D = 128, 128
    kv_elem = 1 if prob["kv_fp8"] else 2
    ro = prob["row_off"].cpu().tolist()
    L = prob["kv_lens"]
    ids = block_ids.cpu().numpy()
    cnt = num_selected.cpu().numpy()
    idx_bytes = sum(L[b] for b in range(prob["batch"]) if ro[b + 1] > ro[b]) * \
        prob["H_idxk"] * D * 2 + prob["total_q"] * prob["H_kv"] * D * 2
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
    """A bounded sample of a workload for the CPU oracle, and its description.  Decode-like
    workloads: n_seq of their sequences (same distributions).  Prefill: one sequence with 16-64
    new tokens over a prior cache drawn as in the workload (a whole prefill sequence is minutes
    of fp64 work per pass)."""
    from block_sparse_paged_scores_b200 import workload as wl
    spec = wl.WORKLOADS[workload]
    q_hi = spec.q_len[1] if isinstance(spec.q_len, tuple) else spec.q_len
    if q_hi > 8:
        p = wl.generate(spec.scaled(batch=1, q_len=(16, 64)), seed=seed)
        desc = (f"1 of {spec.batch} sequences of {workload} with {p['total_q']} new tokens "
                f"(16-64 instead of the workload's q_len; prior cache as in the workload)")
    else:
        p = wl.generate(spec.scaled(batch=min(n_seq, spec.batch)), seed=seed)
        desc = f"{p['batch']} of {spec.batch} sequences of {workload} (same distributions)"
    return p, desc


def time_oracle(prob, min_seconds: float, max_seconds: float):
    import oracle
    oracle.build()
    tokens, t0, reps = 0, time.perf_counter(), 0
    while True:
        oracle.forward(prob, prob["top_k"], prob["init_blocks"], prob["local_blocks"],
                       prob["scale"], prob["max_blocks"])
        tokens += prob["total_q"]
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el * (reps + 1) / reps > max_seconds:
            return tokens / el, el, reps


def cpu_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ arms
def run_reference(args):
    """The CPU oracle as the reference arm: each step is the whole path on a bounded sample
    of the workload (a few of its sequences, same distributions)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    prob, desc = oracle_sample(args.workload, args.cpu_sample_seqs, seed=7)
    import oracle
    oracle.build()
    fwd = lambda: oracle.forward(prob, prob["top_k"], prob["init_blocks"], prob["local_blocks"],
                                 prob["scale"], prob["max_blocks"])
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

    spec = wl.WORKLOADS[args.workload]
    if args.batch:
        spec = spec.scaled(batch=args.batch)
    seed = wl.SEEDS[args.workload] + 1000 * rank
    prob = wl.generate(spec, seed=seed, device=dev)
    path = msa.Path(prob, num_splits=args.splits)
    stream = torch.cuda.current_stream(dev)
    fp8 = prob["kv_fp8"]
    stream_route = prob["max_q_len"] <= 8  # decode / speculative: persistent kernel + combine
    splits_used = msa.msa_attn_partials(path.rp, prob["S"], prob["H_q"], prob["H_kv"],
                                        path.max_blocks, args.splits)[0] if stream_route else 1
    # decode: index, attention with the selection inside, [combine: only with more than one
    # split-K partition]; speculative: index, select, plan, attention, [combine];
    # prefill: index, select, plan, attention
    if prob["max_q_len"] == 1 and prob["H_q"] // prob["H_kv"] <= 16:
        kernels_per_step = 2 + (1 if splits_used > 1 else 0)
    elif stream_route:
        kernels_per_step = 4 + (1 if splits_used > 1 else 0)
    else:
        kernels_per_step = 4

    for _ in range(args.warmup):
        path.run(stream)
    torch.cuda.synchronize(dev)
    assert int(path.dev_err.item()) == 0, "device error flag set during warm-up"

    sampler = ClockSampler(local).start() if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    # a step that touches less than L2 is timed cold: L2 is flushed (a write of twice its size)
    # before every step, outside the step's own events
    idx_bytes, attn_bytes = algorithmic_bytes(prob, path.block_ids, path.num_selected)
    flush = idx_bytes + attn_bytes < L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None

    # ---- device-timed region: exactly K steps between barriers
    barrier(ws, dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    if flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a_, b_ in evs:
            flush_buf.fill_(1)
            a_.record(stream)
            path.run(stream)
            b_.record(stream)
        torch.cuda.synchronize(dev)
        ms_local = sum(a_.elapsed_time(b_) for a_, b_ in evs)
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            path.run(stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_local = e0.elapsed_time(e1)
    barrier(ws, dev)
    t_wall1 = time.time()
    ms = max_over_ranks(ms_local, ws, dev)

    # ---- per-stage durations (separate K-step passes, events between the launches)
    def stage_pass(fns):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
               for _ in range(args.steps)]
        for k in range(args.steps):
            evs[k][0].record(stream)
            for i, fn in enumerate(fns):
                fn()
                evs[k][i + 1].record(stream)
        torch.cuda.synchronize(dev)
        return [sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)) /
                args.steps for i in range(len(fns))]

    attn_key = "attention" + ("_incl_plan" if prob["max_q_len"] > 1 else "")
    if stream_route and splits_used > 1:
        st = stage_pass([lambda: path.index_scores(stream), lambda: path.select(stream=stream),
                         lambda: path.attend(stream=stream, combine=False),
                         lambda: path.combine(stream)])
        stages = {"index_scores": st[0], "select": st[1], attn_key: st[2], "combine": st[3]}
    elif stream_route:  # one partition: the attention kernel writes the output, no combine
        st = stage_pass([lambda: path.index_scores(stream), lambda: path.select(stream=stream),
                         lambda: path.attend(stream=stream)])
        stages = {"index_scores": st[0], "select": st[1], attn_key: st[2]}
    if stream_route:
        # the first two stages as one msa_index_select launch, and the last two (with the
        # combine) as one msa_select_sparse_attn_paged call, for comparison
        stages["fused_index_select"] = stage_pass([lambda: path.index_select(stream)])[0]
        stages["select_in_attention"] = stage_pass([lambda: path.select_attend(stream)])[0]
        stages["step_with_separate_select"] = stage_pass(
            [lambda: (path.index_scores(stream), path.select(stream=stream),
                      path.attend(stream=stream))])[0]
        idx_kind, idx_src = "index_scores", ("indexer.cu", "select_row.cuh")
    else:
        st = stage_pass([lambda: path.index_scores(stream), lambda: path.select(stream=stream),
                         lambda: path.attend(stream=stream)])
        stages = {"index_scores": st[0], "select": st[1], attn_key: st[2]}
        idx_kind, idx_src = "index_scores", ("indexer_tc.cu",)
    idx_ms, attn_ms = st[0], stages[attn_key]
    if sampler:
        sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None

    # ---- end to end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and its output back, both inside the timed region.  The pipelined
    # figure (HostPipeline, two deep) is the headline; the serial one (copy in, compute, copy
    # out on one stream) is reported beside it.
    e2e_ms = e2e_serial_ms = None
    h2d = d2h = 0
    if not args.no_e2e:
        host = {k: prob[k].cpu().pin_memory() for k in msa.HostPipeline.PER_STEP}
        outs = [torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = outs[0].numel() * outs[0].element_size()
        for _ in range(max(1, args.warmup)):
            for k_, v_ in host.items():
                prob[k_].copy_(v_, non_blocking=True)
            path.run(stream)
            outs[0].copy_(path.out, non_blocking=True)
        torch.cuda.synchronize(dev)
        barrier(ws, dev)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(args.steps):
            for k_, v_ in host.items():
                prob[k_].copy_(v_, non_blocking=True)
            path.run(stream)
            outs[0].copy_(path.out, non_blocking=True)
        x1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_serial_ms = max_over_ranks(x0.elapsed_time(x1), ws, dev)

        pipe = msa.HostPipeline(prob, num_splits=args.splits)
        packed = pipe.pack(host)  # the step's inputs as one pinned buffer: one copy per step
        for i in range(max(2, args.warmup)):
            pipe.submit(packed, outs[i % 2])
        pipe.finish(stream)
        torch.cuda.synchronize(dev)
        barrier(ws, dev)
        x0.record(stream)
        pipe.start(after=x0)
        for i in range(args.steps):
            pipe.submit(packed, outs[i % 2])
        pipe.finish(stream)
        x1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(x0.elapsed_time(x1), ws, dev)
        h2d = packed.numel()
        for p_ in pipe.paths:
            assert int(p_.dev_err.item()) == 0, "device error flag set (host pipeline)"
        assert torch.equal(outs[(args.steps - 1) % 2].to(dev), path.out), \
            "host pipeline output differs from the device-resident step"
        del pipe

    # ---- the realised work of this step, for the roofline (idx_bytes, attn_bytes above)
    tokens_total = sum_over_ranks(prob["total_q"], ws, dev) * args.steps
    assert int(path.dev_err.item()) == 0, "device error flag set"

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        sample, desc = oracle_sample(args.workload, args.cpu_sample_seqs, seed=7)
        v, el, reps = time_oracle(sample, args.cpu_min_s, args.cpu_max_s)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{desc}, seed 7, {reps} pass(es), {el:.1f} s"}

    if rank != 0:
        return 0
    hbm, bf16, bf16_sus, peak_src = measured_peaks()
    tensor_route = prob["max_q_len"] > 8  # prefill: dense contractions on the tensor cores
    kinds = {idx_kind: (idx_ms, idx_bytes, idx_src),
             "attention": (attn_ms, attn_bytes,
                           ("attention_stream.cu", "attn_common.cuh", "select_row.cuh")
                           if stream_route else
                           (("attention_tile.cu", "attn_common.cuh") if fp8
                            else ("attention_tc.cu",)))}
    dom = max(kinds, key=lambda k: kinds[k][0])
    d_ms, d_bytes, d_src = kinds[dom]
    digest = source_digest(*d_src)
    if tensor_route:
        idx_flops, attn_flops = algorithmic_flops(prob, path.block_ids, path.num_selected)
        d_flops = attn_flops if dom == "attention" else idx_flops
        achieved = d_flops / (d_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": bf16,
                    "unit": "TFLOP/s", "frac": achieved / bf16, "peak_source": peak_src,
                    "traffic": profiled_traffic(dom, args.workload, digest),
                    "algorithmic_flops_per_launch": d_flops,
                    "note": "algorithmic FLOPs (selected, causally clipped positions only) over "
                            "the kernel's time, against the bf16 burst peak"}
        if dom == "attention" and not fp8:
            ex = executed_flops_tiles(prob, path.block_ids, path.num_selected,
                                      128 // (prob["H_q"] // prob["H_kv"]))
            roofline["executed_flops_per_launch"] = ex
            roofline["executed_tflops"] = ex / (d_ms * 1e-3) / 1e12
            roofline["executed_frac"] = ex / (d_ms * 1e-3) / 1e12 / bf16
    else:
        achieved = d_bytes / (d_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                    "unit": "GB/s", "frac": achieved / hbm, "peak_source": peak_src,
                    "traffic": profiled_traffic(dom, args.workload, digest),
                    "algorithmic_bytes_per_launch": d_bytes}
    line = {
        "metric": METRIC, "value": tokens_total / (ms * 1e-3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 kv / bf16" if fp8 else "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": prob["batch"],
                   "q_tokens_per_step": prob["total_q"], "H_kv": prob["H_kv"],
                   "H_q": prob["H_q"], "head_dim": 128, "page_size": 128,
                   "top_k": prob["top_k"], "init_blocks": prob["init_blocks"],
                   "local_blocks": prob["local_blocks"], "kv_lens": f"{spec.kv_len}",
                   "split_k_partials": splits_used, "parallelism": f"replicas x{ws}",
                   "l2": (f"{(idx_bytes + attn_bytes) / 2**20:.1f} MiB touched per step, under "
                          f"the {L2_BYTES / 2**20:.0f} MiB L2: L2 flushed before every step (a "
                          f"{2 * L2_BYTES / 2**20:.0f} MiB write outside the step's events), "
                          f"time = sum of the steps' own intervals") if flush else
                         (f"inputs larger than L2: {(idx_bytes + attn_bytes) / 2**20:.0f} MiB "
                          f"touched per step vs {L2_BYTES / 2**20:.0f} MiB L2, no flush")},
        "roofline": roofline,
        "step_hbm": {"algorithmic_bytes": idx_bytes + attn_bytes,
                     "achieved_GBps": (idx_bytes + attn_bytes) / (ms / args.steps * 1e-3) / 1e9,
                     "frac_of_measured": (idx_bytes + attn_bytes) / (ms / args.steps * 1e-3)
                     / 1e9 / hbm,
                     "frac_of_8TBps": (idx_bytes + attn_bytes) / (ms / args.steps * 1e-3)
                     / 8e12},
        "stages_ms": stages,
        "gpu_launches": kernels_per_step * args.steps,
        "clocks": clocks,
        "e2e": None if e2e_ms is None else {
            "value": tokens_total / (e2e_ms * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "serial_value": tokens_total / (e2e_serial_ms * 1e-3),
            "note": "per-step inputs (q, q_idx, row offsets, cache lengths, page table) copied "
                    "from pinned host memory and the output read back, every step inside the "
                    "timed region; value: two-deep pipeline (the step's inputs packed in one "
                    "pinned buffer, one copy; step i+1's copy in and step i-1's copy out on "
                    "their own streams while step i computes); serial_value: one copy per "
                    "input, compute, copy out, all on one stream; the caches stay resident"},
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="bf16_decode")
    ap.add_argument("--splits", type=int, default=0, help="split-K partitions (0 = heuristic)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch "
                    "(profiling runs on a smaller case; not a bench number)")
    ap.add_argument("--cpu-sample-seqs", type=int, default=4)
    ap.add_argument("--cpu-min-s", type=float, default=10.0)
    ap.add_argument("--cpu-max-s", type=float, default=30.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    rc = run_ours(args)
    ws, _, _ = dist_env()
    if ws > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
