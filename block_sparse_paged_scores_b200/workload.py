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
     last page, is set to NaN (bf16 0x7FC0, e4m3 0x7F) so that a stray read shows up;
  5. a scaled index-K cache ("fp8" / "fp4" index dtype) is the N(0,1) index-K of step 3,
     quantised: fp8 with one float32 scale per token (its largest |value| / 448, then each
     element rounded to e4m3), fp4 with one UE8M0 exponent per 32 elements (the smallest
     2^e with largest |value| / 2^e <= 6, then each element rounded to the nearest E2M1
     value); poisoned positions get a NaN scale (fp8) or the NaN exponent 0xFF (fp4).

Layouts (the C-ABI's):
  q      bf16 [total_q, H_q, 128]         q_idx  bf16 [total_q, H_kv, 128]
  k_idx  bf16 [num_pages, H_idxk, 128, 128], or for a scaled index-K cache
         fp8: uint8 e4m3 codes [num_pages, H_idxk, 128, 128] + k_idx_scale f32 [.., 128]
         fp4: uint8 e2m1 pairs [num_pages, H_idxk, 128, 64] + k_idx_scale u8 [.., 128, 4]
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
    idx_dtype: str = "bf16"    # index-K cache: "bf16" | "fp8" (e4m3 + f32 scale per token)
                               # | "fp4" (e2m1 + ue8m0 exponent per 32 elements)
    q_idx_window: int = 0      # > 1: each sequence's index queries are the moving average of
                               # that many consecutive N(0,1) draws (times sqrt(window): unit
                               # variance), so that neighbouring tokens' queries are coherent

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


# E2M1 magnitudes by code and the midpoints between neighbours (a value on a midpoint goes to
# the lower code)
_E2M1_MID = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def quantize_index_k(x: torch.Tensor, idx_dtype: str, chunk_pages: int = 4096):
    """(codes, scales) of an index-K cache ``x`` (bf16 [pages, H, 128, 128]) in the scaled
    format ``idx_dtype``, computed on x's device page-chunk by page-chunk."""
    P, H = x.shape[0], x.shape[1]
    dev = x.device
    if idx_dtype == "fp8":
        codes = torch.empty((P, H, BLOCK, HEAD_DIM), dtype=torch.uint8, device=dev)
        scales = torch.empty((P, H, BLOCK), dtype=torch.float32, device=dev)
    else:
        codes = torch.empty((P, H, BLOCK, HEAD_DIM // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((P, H, BLOCK, HEAD_DIM // 32), dtype=torch.uint8, device=dev)
        mids = torch.tensor(_E2M1_MID, dtype=torch.float32, device=dev)
    for s in range(0, P, chunk_pages):
        e = min(P, s + chunk_pages)
        v = x[s:e].float()
        if idx_dtype == "fp8":
            amax = v.abs().amax(-1)
            sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            codes[s:e] = (v / sc[..., None]).clamp(-448.0, 448.0).to(
                torch.float8_e4m3fn).view(torch.uint8)
            scales[s:e] = sc
        else:
            g = v.reshape(e - s, H, BLOCK, HEAD_DIM // 32, 32)
            amax = g.abs().amax(-1)
            ex = torch.ceil(torch.log2(torch.clamp(amax / 6.0, min=2.0 ** -126)))
            ex = torch.clamp(ex, -126, 127)
            y = g / torch.exp2(ex)[..., None]
            mag = torch.bucketize(y.abs().clamp(max=6.0), mids).to(torch.uint8)   # 0..7
            code = mag | ((y < 0).to(torch.uint8) << 3)
            code = code.reshape(e - s, H, BLOCK, HEAD_DIM // 2, 2)
            codes[s:e] = code[..., 0] | (code[..., 1] << 4)
            scales[s:e] = (ex + 127).to(torch.uint8)
    return codes, scales


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
    q_idx = torch.randn((total_q, spec.H_kv, HEAD_DIM), generator=gdev, device=device)
    if spec.q_idx_window > 1:
        w = spec.q_idx_window
        coh = torch.empty_like(q_idx)
        for b in range(spec.batch):
            r0, r1 = int(row_off[b]), int(row_off[b + 1])
            if r1 == r0:
                continue
            e = torch.randn((r1 - r0 + w - 1, spec.H_kv, HEAD_DIM), generator=gdev,
                            device=device, dtype=torch.float64)
            c = torch.cat([torch.zeros_like(e[:1]), torch.cumsum(e, 0)])
            coh[r0:r1] = ((c[w:] - c[:-w]) / math.sqrt(w)).float()
        q_idx = coh
    q_idx = q_idx.to(bf16)
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

    k_idx_scale = None
    if spec.idx_dtype != "bf16":
        k_idx, k_idx_scale = quantize_index_k(k_idx, spec.idx_dtype)
        if poison:
            # the NaN scale / exponent reaches every element of a poisoned token
            bad = 0xFF if spec.idx_dtype == "fp4" else float("nan")
            if unused.numel():
                k_idx_scale[unused] = bad
            for b in range(spec.batch):
                tail = int(L[b]) % BLOCK
                if tail:
                    last = int(table[b, int(nb[b]) - 1])
                    k_idx_scale[last, :, tail:] = bad

    return dict(
        name=spec.name, spec=spec, seed=seed,
        row_off=row_off.to(device), cache_len=cache_len.to(torch.int32).to(device),
        table=table.to(device), q=q, q_idx=q_idx, k_idx=k_idx, k_idx_scale=k_idx_scale,
        idx_dtype=spec.idx_dtype, k=k, v=v,
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


# ------------------------------------------------------------------ latent sparse attention
@dataclasses.dataclass(frozen=True)
class LatentSpec:
    """A workload of the latent sparse attention op (Mojo
    Struct_latent_sparse_attention_ragged_paged): a K = V latent (128 wide, shared by the H
    query heads) in two paged leaves with a layer axis, a sliding window over one and a
    per-query entry list into the other, a per-head sink."""
    name: str
    batch: int
    q_len: IntOrRange
    H: int
    window: int
    n_entries: int
    swa_len: IntOrRange        # prior tokens of the sliding-window leaf (new ones follow)
    comp_len: IntOrRange       # entries of the compressed leaf
    layers: int = 2
    layer: int = 1

    def scaled(self, **kw) -> "LatentSpec":
        return dataclasses.replace(self, **kw)


LATENT_DECODE = LatentSpec("latent_decode", batch=64, q_len=1, H=64, window=128,
                           n_entries=512, swa_len=(1024, 8192), comp_len=(2048, 8192))


def _paged_leaf(lengths, first_needed, layers, gen_cpu, gdev, device, poison):
    """A paged leaf holding positions [first_needed[b], lengths[b]) of every sequence (pages
    below the first needed one are left out of the table, -1), N(0,1) bf16 values, the pool
    shuffled; unused pool pages and positions past a sequence's end are NaN."""
    batch = len(lengths)
    nb = [(int(L) + BLOCK - 1) // BLOCK for L in lengths]
    lo = [int(f) // BLOCK for f in first_needed]
    total = sum(n - l for n, l in zip(nb, lo))
    pool = max(total, 1)
    perm = torch.randperm(pool, generator=gen_cpu)
    max_pages = max(1, max(nb))
    table = torch.full((batch, max_pages), -1, dtype=torch.int32)
    cur = 0
    for b in range(batch):
        for j in range(lo[b], nb[b]):
            table[b, j] = int(perm[cur])
            cur += 1
    kv = _normal_pages((pool, layers, BLOCK, HEAD_DIM), gdev, device, torch.bfloat16)
    if poison:
        unused = perm[total:].to(device)
        if unused.numel():
            kv[unused] = float("nan")
        for b in range(batch):
            tail = int(lengths[b]) % BLOCK
            if tail:
                kv[int(table[b, nb[b] - 1]), :, tail:] = float("nan")
    return kv, table


def generate_latent(spec: LatentSpec, seed: int, device="cpu", poison: bool = True) -> dict:
    """One seeded latent problem.  Draw order: lengths (new tokens, window-leaf prior, compressed
    leaf), the window leaf's page permutation, the compressed leaf's, each query's entry list
    (a uniform random subset of its sequence's compressed entries, ascending, -1 padded when
    the leaf is shorter than n_entries), then q, the window leaf, the compressed leaf and the
    sinks as N(0,1)."""
    gcpu = torch.Generator().manual_seed(seed)
    q_lens = _draw(spec.q_len, spec.batch, gcpu)
    swa_prior = _draw(spec.swa_len, spec.batch, gcpu)
    comp_len = _draw(spec.comp_len, spec.batch, gcpu)
    L_swa = swa_prior + q_lens
    first = torch.clamp(swa_prior - spec.window + 1, min=0)
    row_off = torch.zeros(spec.batch + 1, dtype=torch.int32)
    row_off[1:] = torch.cumsum(q_lens, 0).to(torch.int32)
    total_q = int(row_off[-1])
    gdev = torch.Generator(device=device).manual_seed(seed)
    swa_kv, swa_table = _paged_leaf(L_swa.tolist(), first.tolist(), spec.layers, gcpu, gdev,
                                    device, poison)
    comp_kv, comp_table = _paged_leaf(comp_len.tolist(), [0] * spec.batch, spec.layers, gcpu,
                                      gdev, device, poison)
    comp_idx = torch.full((total_q, spec.n_entries), -1, dtype=torch.int32)
    for b in range(spec.batch):
        n = min(spec.n_entries, int(comp_len[b]))
        for t in range(int(row_off[b]), int(row_off[b + 1])):
            comp_idx[t, :n] = torch.sort(torch.randperm(int(comp_len[b]), generator=gcpu)[:n])[0]
    q = torch.randn((total_q, spec.H, HEAD_DIM), generator=gdev, device=device).to(torch.bfloat16)
    sink = torch.randn((spec.H,), generator=gdev, device=device, dtype=torch.float32)
    return dict(
        name=spec.name, spec=spec, seed=seed, batch=spec.batch, total_q=total_q,
        max_q_len=max(1, int(q_lens.max())), H=spec.H, window=spec.window,
        n_entries=spec.n_entries, row_off=row_off.to(device), q=q,
        swa_kv=swa_kv, swa_len=swa_prior.to(torch.int32).to(device),
        swa_table=swa_table.to(device), swa_layer=spec.layer,
        comp_kv=comp_kv, comp_len=comp_len.to(torch.int32).to(device),
        comp_table=comp_table.to(device), comp_layer=spec.layer,
        comp_idx=comp_idx.to(device), sink=sink, scale=1.0 / math.sqrt(HEAD_DIM),
        q_lens=q_lens.tolist(), swa_lens=L_swa.tolist(), comp_lens=comp_len.tolist())
