"""Seeded synthetic workloads for block-sparse paged attention.

This module only draws inputs: lengths, a shuffled page table and N(0,1) tensors laid out in
the paged cache format.  It holds none of the method's arithmetic (no scores, no selection,
no softmax), so the GPU path, the tests and the CPU oracle can all consume its output.

Recipe (all draws from ``torch.Generator`` seeded with the workload's seed, in this order):
  1. per-sequence new-query lengths and KV lengths (CPU generator);
  2. a random permutation of the page pool; sequence b's logical block j gets the next
     page of the permutation (CPU generator);
  3. q, q_idx, k_idx, K, V as standard normals on the target device, rounded to bf16 (RNE),
     or for e4m3 KV clamped to +-448 and cast with torch's float8_e4m3fn (RNE);
  4. poison: every pool page no sequence uses, and every position >= L_b of a sequence's
     last page, is set to NaN (bf16 0x7FC0, e4m3 0x7F) so that a stray read shows up.

Layouts (the C-ABI's):
  q      bf16 [total_q, H_q, 128]         q_idx  bf16 [total_q, H_kv, 128]
  k_idx  bf16 [num_pages, H_idxk, 128, 128]
  k, v   bf16 | float8_e4m3fn [num_pages, H_kv, 128, 128]
  row_off int32 [batch+1], cache_len int32 [batch], table int32 [batch, max_pages] (-1 unused)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple, Union

import torch

BLOCK = 128
HEAD_DIM = 128

IntOrRange = Union[int, Tuple[int, int]]


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    batch: int
    q_len: IntOrRange          # new query tokens per sequence (fixed or uniform [lo, hi])
    kv_len: IntOrRange         # L_b including the new tokens, unless ``prior_len`` is given
    H_kv: int
    G: int                     # query heads per KV head
    top_k: int
    init_blocks: int
    local_blocks: int
    kv_dtype: str = "bf16"     # "bf16" | "fp8"
    H_idxk: int = 1            # index-K heads: 1 (shared) or H_kv
    prior_len: Optional[IntOrRange] = None   # prefill: prior cache length, L_b = prior + q_len
    pool_pages: int = 0        # minimum pool size (extra pages stay unused and poisoned)

    @property
    def H_q(self) -> int:
        return self.H_kv * self.G

    @property
    def S(self) -> int:
        return self.init_blocks + self.local_blocks + self.top_k

    def scaled(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


# The five workloads the method is measured on.
TINY_DECODE = WorkloadSpec("tiny_decode", batch=1, q_len=1, kv_len=1024, H_kv=1, G=4, top_k=4,
                           init_blocks=1, local_blocks=1, pool_pages=16)
BF16_DECODE = WorkloadSpec("bf16_decode", batch=32, q_len=1, kv_len=(16384, 65536), H_kv=8, G=8,
                           top_k=16, init_blocks=1, local_blocks=2)
SPEC_DECODE = WorkloadSpec("spec_decode", batch=64, q_len=4, kv_len=(8192, 32768), H_kv=8, G=8,
                           top_k=32, init_blocks=1, local_blocks=2)
FP8_LONG_DECODE = WorkloadSpec("fp8_long_decode", batch=128, q_len=1, kv_len=131072, H_kv=8, G=8,
                               top_k=64, init_blocks=1, local_blocks=4, kv_dtype="fp8")
RAGGED_PREFILL = WorkloadSpec("ragged_prefill", batch=8, q_len=(512, 4096), kv_len=0,
                              prior_len=(0, 32768), H_kv=8, G=8, top_k=64, init_blocks=1,
                              local_blocks=2)

WORKLOADS = {w.name: w for w in (TINY_DECODE, BF16_DECODE, SPEC_DECODE, FP8_LONG_DECODE,
                                 RAGGED_PREFILL)}
SEEDS = {"tiny_decode": 1, "bf16_decode": 2, "spec_decode": 3, "fp8_long_decode": 4,
         "ragged_prefill": 5}


def _draw(r: IntOrRange, n: int, gen: torch.Generator) -> torch.Tensor:
    if isinstance(r, int):
        return torch.full((n,), r, dtype=torch.int64)
    lo, hi = r
    return torch.randint(lo, hi + 1, (n,), generator=gen, dtype=torch.int64)


def _normal_pages(shape, gen, device, dtype, chunk_elems=1 << 25):
    """Pool tensor of N(0,1) values drawn chunk by chunk along dim 0 (bounds temporaries)."""
    out = torch.empty(shape, dtype=dtype, device=device)
    per = max(1, chunk_elems // max(1, math.prod(shape[1:])))
    for s in range(0, shape[0], per):
        e = min(shape[0], s + per)
        x = torch.randn((e - s,) + tuple(shape[1:]), generator=gen, device=device,
                        dtype=torch.float32)
        if dtype == torch.float8_e4m3fn:
            x.clamp_(-448.0, 448.0)
        out[s:e] = x.to(dtype)
    return out


def _fill_nan(t: torch.Tensor, index):
    if t.dtype == torch.float8_e4m3fn:
        t.view(torch.uint8)[index] = 0x7F
    else:
        t[index] = float("nan")


def generate(spec: WorkloadSpec, seed: int, device="cpu", poison: bool = True) -> dict:
    """Draw one seeded problem for ``spec``; tensors live on ``device``."""
    gcpu = torch.Generator().manual_seed(seed)
    q_lens = _draw(spec.q_len, spec.batch, gcpu)
    if spec.prior_len is not None:
        prior = _draw(spec.prior_len, spec.batch, gcpu)
        L = prior + q_lens
    else:
        L = _draw(spec.kv_len, spec.batch, gcpu)
    assert bool((L >= q_lens).all()) and bool((q_lens >= 0).all())
    cache_len = L - q_lens
    nb = (L + BLOCK - 1) // BLOCK
    total_pages = int(nb.sum())
    pool = max(total_pages, spec.pool_pages)
    perm = torch.randperm(pool, generator=gcpu)
    max_pages = max(1, int(nb.max()))
    table = torch.full((spec.batch, max_pages), -1, dtype=torch.int32)
    cur = 0
    for b in range(spec.batch):
        n = int(nb[b])
        table[b, :n] = perm[cur:cur + n].to(torch.int32)
        cur += n
    row_off = torch.zeros(spec.batch + 1, dtype=torch.int32)
    row_off[1:] = torch.cumsum(q_lens, 0).to(torch.int32)
    total_q = int(row_off[-1])

    gdev = torch.Generator(device=device).manual_seed(seed)
    bf16 = torch.bfloat16
    kvt = torch.float8_e4m3fn if spec.kv_dtype == "fp8" else bf16
    q = torch.randn((total_q, spec.H_q, HEAD_DIM), generator=gdev, device=device).to(bf16)
    q_idx = torch.randn((total_q, spec.H_kv, HEAD_DIM), generator=gdev, device=device).to(bf16)
    k_idx = _normal_pages((pool, spec.H_idxk, BLOCK, HEAD_DIM), gdev, device, bf16)
    k = _normal_pages((pool, spec.H_kv, BLOCK, HEAD_DIM), gdev, device, kvt)
    v = _normal_pages((pool, spec.H_kv, BLOCK, HEAD_DIM), gdev, device, kvt)

    if poison:
        unused = perm[total_pages:].to(device)
        if unused.numel():
            for t in (k_idx, k, v):
                _fill_nan(t, unused)
        for b in range(spec.batch):
            tail = int(L[b]) % BLOCK
            if tail:
                last = int(table[b, int(nb[b]) - 1])
                for t in (k_idx, k, v):
                    _fill_nan(t, (last, slice(None), slice(tail, None)))

    return dict(
        name=spec.name, spec=spec, seed=seed,
        row_off=row_off.to(device), cache_len=cache_len.to(torch.int32).to(device),
        table=table.to(device), q=q, q_idx=q_idx, k_idx=k_idx, k=k, v=v,
        kv_fp8=spec.kv_dtype == "fp8",
        batch=spec.batch, total_q=total_q, max_q_len=max(1, int(q_lens.max())),
        max_cache_len=int(cache_len.max()), max_pages=max_pages, num_pages=max(pool, 1),
        max_blocks=max_pages, H_q=spec.H_q, H_kv=spec.H_kv, H_idxk=spec.H_idxk,
        top_k=spec.top_k, init_blocks=spec.init_blocks, local_blocks=spec.local_blocks,
        S=spec.S, scale=1.0 / math.sqrt(HEAD_DIM), kv_lens=L.tolist(), q_lens=q_lens.tolist(),
    )


def to_device(prob: dict, device) -> dict:
    """Copy every tensor of a problem to ``device`` (same bytes)."""
    out = {}
    for k_, v_ in prob.items():
        out[k_] = v_.to(device) if isinstance(v_, torch.Tensor) else v_
    return out
