"""Comparison helpers shared by the GPU parity tests (imported by tests only).

Tolerances:
- block scores: the GPU accumulates exact bf16 products in fp32 over 128 dims; the error of a
  128-term fp32 sum is below 128 * 2^-24 * sum_c |q_c k_c| <= 2^-17 * ||q|| * ||k|| (Cauchy-
  Schwarz).  The check allows 2^-15 * ||q_idx|| * max_pos ||k_idx[pos]|| per (row, head, block)
  and requires the -inf pattern (blocks a query cannot see) to match exactly.
- selection: ids must match bit for bit wherever the top_k-th and (top_k+1)-th candidate
  scores differ by more than 1e-3 relative; elsewhere the GPU set must be a valid top-k under
  the oracle's scores up to that same tolerance.  Run on identical fp32 scores, the GPU and the
  oracle selections must match bit for bit everywhere.
- attention: max |diff| <= 2e-2 and mean |diff| <= 2e-3 for BF16 KV, max |diff| <= 6e-2 for
  FP8 KV, against the oracle's fp64 result.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

BLOCK = 128
SCORE_TOL_FACTOR = 2.0 ** -15
REL_GAP = 1e-3
ATTN_TOL = {False: (2e-2, 2e-3), True: (6e-2, 6e-3)}


def dequantized_index_k(prob) -> torch.Tensor:
    """The index-K cache of ``prob`` as fp32 values [num_pages, H_idxk, 128, 128], decoded with
    library routines (torch for bf16, e4m3 and e8m0, ml_dtypes for e2m1)."""
    dt = prob.get("idx_dtype", "bf16")
    codes = prob["k_idx"].cpu()
    if dt == "bf16":
        return codes.float()
    sc = prob["k_idx_scale"].cpu()
    if dt == "fp8":
        return codes.view(torch.float8_e4m3fn).float() * sc[..., None]
    import ml_dtypes
    c = codes.numpy()
    lo = (c & 15).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    hi = (c >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    v = torch.from_numpy(np.stack([lo, hi], axis=-1).reshape(c.shape[:3] + (128,)))
    ex = sc.view(torch.float8_e8m0fnu).float()
    return v * ex.repeat_interleave(32, dim=-1)


def block_key_norms(prob) -> np.ndarray:
    """max over each block's positions of ||k_idx[pos]||: [batch, H_idxk, max_blocks]
    (positions >= L_b excluded)."""
    kn = torch.nan_to_num(dequantized_index_k(prob), nan=0.0).norm(dim=-1)  # [pool, H, 128]
    table = prob["table"].long().clamp(min=0)
    out = kn[table].amax(dim=-1)                                          # [batch, max_pages, H]
    return out.permute(0, 2, 1).cpu().numpy()


def check_scores(gpu, orc, prob, max_blocks):
    gpu = np.asarray(gpu, dtype=np.float64)
    orc = np.asarray(orc, dtype=np.float64)
    assert gpu.shape == orc.shape
    inf_o, inf_g = np.isneginf(orc), np.isneginf(gpu)
    assert np.array_equal(inf_o, inf_g), "visible-block pattern differs"
    assert not np.isnan(gpu).any()
    qn = prob["q_idx"].float().norm(dim=-1).cpu().numpy()                 # [tq, H_kv]
    kn = block_key_norms(prob)                                            # [b, H_idxk, mb]
    ro = prob["row_off"].cpu().tolist()
    H_kv, H_idxk = prob["H_kv"], prob["H_idxk"]
    worst = 0.0
    for b in range(prob["batch"]):
        for t in range(ro[b], ro[b + 1]):
            for g in range(H_kv):
                fin = ~inf_o[t, g]
                tol = SCORE_TOL_FACTOR * qn[t, g] * kn[b, g % H_idxk, :max_blocks][fin] + 1e-30
                err = np.abs(gpu[t, g, fin] - orc[t, g, fin])
                assert np.all(err <= tol), (t, g, float(err.max()), float(tol.min()))
                if err.size:
                    worst = max(worst, float((err / tol).max()))
    return worst


def _visible(prob):
    ro = prob["row_off"].cpu().tolist()
    cl = prob["cache_len"].cpu().tolist()
    nb = np.zeros(prob["total_q"], dtype=np.int64)
    for b in range(prob["batch"]):
        for i in range(ro[b + 1] - ro[b]):
            nb[ro[b] + i] = (cl[b] + i) // BLOCK + 1
    return nb


def check_selection(gpu_ids, gpu_cnt, orc_ids, orc_cnt, orc_scores, prob, exact=False):
    """Bit-exact where the cut is separated by more than REL_GAP (everywhere if ``exact``);
    otherwise a valid top-k under the oracle scores.  Returns a boolean [tq, H_kv] mask of the
    rows whose ids are identical."""
    gpu_ids, gpu_cnt = np.asarray(gpu_ids), np.asarray(gpu_cnt)
    orc_ids, orc_cnt = np.asarray(orc_ids), np.asarray(orc_cnt)
    nbv = _visible(prob)
    init, local, top_k = prob["init_blocks"], prob["local_blocks"], prob["top_k"]
    same = np.zeros(gpu_cnt.shape, dtype=bool)
    for t in range(gpu_cnt.shape[0]):
        nb = int(nbv[t])
        forced = [j for j in range(nb) if j < init or j >= nb - local]
        cand = np.array([j for j in range(nb) if j not in set(forced)], dtype=np.int64)
        for g in range(gpu_cnt.shape[1]):
            gi = gpu_ids[t, g, :gpu_cnt[t, g]].tolist()
            oi = orc_ids[t, g, :orc_cnt[t, g]].tolist()
            assert all(x == -1 for x in gpu_ids[t, g, gpu_cnt[t, g]:])
            if gi == oi:
                same[t, g] = True
                continue
            assert not exact, (t, g, gi, oi)
            s = orc_scores[t, g, cand]
            order = np.sort(s)[::-1]
            assert len(cand) > top_k
            sk, sk1 = order[top_k - 1], order[top_k]
            tol = REL_GAP * abs(sk)
            assert sk - sk1 <= tol, (t, g, gi, oi, sk, sk1)
            # the GPU set is still a valid selection up to the tie tolerance
            assert gi == sorted(set(gi)) and set(forced) <= set(gi)
            assert len(gi) == len(oi)
            kept = [orc_scores[t, g, j] for j in gi if j not in forced]
            dropped = [orc_scores[t, g, j] for j in cand if j not in gi]
            assert min(kept) >= sk - tol and max(dropped) <= sk + tol
    return same


def check_attention(gpu_out, orc_out, fp8, rows_mask=None):
    g = torch.as_tensor(gpu_out).double().cpu().numpy()
    o = np.asarray(orc_out, dtype=np.float64)
    assert not np.isnan(g).any()
    if rows_mask is not None:
        g, o = g[rows_mask], o[rows_mask]
    if g.size == 0:
        return 0.0, 0.0
    d = np.abs(g - o)
    max_tol, mean_tol = ATTN_TOL[bool(fp8)]
    assert d.max() <= max_tol, float(d.max())
    if not fp8:
        assert d.mean() <= mean_tol, float(d.mean())
    return float(d.max()), float(d.mean())


def head_rows_mask(same, G):
    """[tq, H_q] mask of query heads whose KV head's selection matched."""
    return np.repeat(same, G, axis=1)


def single_row_problem(prob, t):
    """The query row t of ``prob`` as a one-token problem on the host: same position, same
    pages (copied into a compact pool), same values.  Rows of the original problem are
    independent of one another, so the oracle's answer for this problem is its answer for
    row t."""
    ro = prob["row_off"].cpu().tolist()
    b = max(i for i in range(prob["batch"]) if ro[i] <= t)
    i = t - ro[b]
    p = int(prob["cache_len"][b]) + i
    nb = p // BLOCK + 1
    pages = prob["table"][b, :nb].long()
    sub = dict(prob)
    sub.update(
        row_off=torch.tensor([0, 1], dtype=torch.int32),
        cache_len=torch.tensor([p], dtype=torch.int32),
        table=torch.arange(nb, dtype=torch.int32)[None],
        q=prob["q"][t:t + 1].cpu(), q_idx=prob["q_idx"][t:t + 1].cpu(),
        k_idx=prob["k_idx"][pages].cpu(), k=prob["k"][pages].cpu(), v=prob["v"][pages].cpu(),
        batch=1, total_q=1, max_q_len=1, max_pages=nb, max_blocks=nb, num_pages=nb)
    return sub


def oracle_forward(prob, max_blocks=None):
    mb = max_blocks or prob["max_blocks"]
    return oracle.forward(prob, prob["top_k"], prob["init_blocks"], prob["local_blocks"],
                          prob["scale"], mb)


def fp32_exact(x):
    """fp64 copy of the fp32 rounding of x (the values a GPU select sees)."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)



# ------------------------------------------------------------------ planted large logits
LOG2E = 1.4426950408889634


def plant_large_keys(prob, every=4, phase=3, factor=16.0):
    """A copy of ``prob`` whose main K rows of every block j with j % every == phase (in each
    sequence's own block order) are multiplied by ``factor`` (a power of two: exact in bf16,
    and in e4m3 for N(0,1) values).  Those blocks then hold logits about ``factor`` times
    larger than the others, so that a row's running maximum jumps far up at a block that
    comes after blocks it has already accumulated."""
    p = dict(prob)
    k = prob["k"].clone()
    table = prob["table"].cpu()
    pages = []
    for b in range(prob["batch"]):
        nb = int((table[b] >= 0).sum())
        pages += [int(table[b, j]) for j in range(phase, nb, every)]
    idx = torch.tensor(sorted(set(pages)), dtype=torch.long, device=k.device)
    if idx.numel():
        k[idx] = (k[idx].float() * factor).to(k.dtype)
    p["k"] = k
    return p


def block_max_logits(prob, ids, cnt):
    """[total_q, H_q, S] largest raw logit q . k over the causally visible positions of each
    selected block (-inf for padding slots), computed densely per sequence in fp32 on the
    problem's device (a check of how the inputs were built, not a reference)."""
    dev = prob["q"].device
    ro = prob["row_off"].cpu().tolist()
    cl = prob["cache_len"].cpu().tolist()
    table = prob["table"].cpu()
    H_q, H_kv = prob["H_q"], prob["H_kv"]
    G = H_q // H_kv
    ids = np.asarray(ids)
    cnt = np.asarray(cnt)
    S = ids.shape[2]
    out = np.full((prob["total_q"], H_q, S), -np.inf)
    for b in range(prob["batch"]):
        n = ro[b + 1] - ro[b]
        if n == 0:
            continue
        L = cl[b] + n
        nb = (L + BLOCK - 1) // BLOCK
        pg = table[b, :nb].long().to(dev)
        kb = prob["k"][pg].float().nan_to_num(0.0)            # [nb, H_kv, 128, 128]
        kb = kb.permute(1, 0, 2, 3).reshape(H_kv, nb * BLOCK, -1)
        q = prob["q"][ro[b]:ro[b + 1]].float().reshape(n, H_kv, G, -1)
        lg = torch.einsum("tgjd,gpd->tgjp", q, kb)             # [n, H_kv, G, nb*128]
        pos = torch.arange(nb * BLOCK, device=dev)
        p_t = cl[b] + torch.arange(n, device=dev)
        lg = lg.masked_fill(pos[None, None, None, :] > p_t[:, None, None, None], -float("inf"))
        bm = lg.reshape(n, H_kv, G, nb, BLOCK).amax(-1).reshape(n, H_q, nb).cpu().numpy()
        for i in range(n):
            t = ro[b] + i
            for h in range(H_q):
                g = h // G
                sel = ids[t, g, :cnt[t, g]]
                out[t, h, :len(sel)] = bm[i, h, sel]
    return out


def lazy_rescale_events(prob, ids, cnt, bmax, tile_tokens, groups, threshold_log2=8.0):
    """How often a row's running maximum moves up by more than 2^threshold_log2 (exp2 domain:
    scale * log2(e) * logit) at a block after one the row has already accumulated, with the
    blocks of each query tile's union of selections dealt out to ``groups`` alternating
    groups (each keeping its own running maximum, moved only past the threshold).  With
    tile_tokens = 1 and groups = 1 that is the row's own list of blocks."""
    ro = prob["row_off"].cpu().tolist()
    H_q, H_kv = prob["H_q"], prob["H_kv"]
    G = H_q // H_kv
    sl2 = prob["scale"] * LOG2E
    ids = np.asarray(ids)
    cnt = np.asarray(cnt)
    events = 0
    for b in range(prob["batch"]):
        for t0 in range(ro[b], ro[b + 1], tile_tokens):
            t1 = min(t0 + tile_tokens, ro[b + 1])
            for g in range(H_kv):
                union = sorted(set(int(j) for t in range(t0, t1)
                                   for j in ids[t, g, :cnt[t, g]]))
                for t in range(t0, t1):
                    own = {int(j): s for s, j in enumerate(ids[t, g, :cnt[t, g]])}
                    for h in range(g * G, (g + 1) * G):
                        m = [-np.inf] * groups
                        for i, j in enumerate(union):
                            if j not in own:
                                continue
                            mb = bmax[t, h, own[j]] * sl2
                            w = i % groups
                            if mb > m[w] + threshold_log2:
                                if np.isfinite(m[w]):
                                    events += 1
                                m[w] = mb
    return events
