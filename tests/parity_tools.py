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


def block_key_norms(prob) -> np.ndarray:
    """max over each block's positions of ||k_idx[pos]||: [batch, H_idxk, max_blocks]
    (positions >= L_b excluded)."""
    kn = torch.nan_to_num(prob["k_idx"].float(), nan=0.0).norm(dim=-1)   # [pool, H_idxk, 128]
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

