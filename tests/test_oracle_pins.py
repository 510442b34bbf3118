"""Pins for the CPU oracle: each test checks it against something other than itself.

- torch's own bf16 and float8_e4m3fn decoders (library routines), all codes;
- numpy brute force of the block score (dense unpaged copy, reshape to blocks, max);
- exhaustive subset search for the selection, hand-worked selection cases
  (tests/golden/select_worked_examples.json) and the selection invariants stated on the
  ferrox-core 'Module block_sparse' page;
- torch.nn.functional.scaled_dot_product_attention in fp64 with an explicit mask (library
  routine) when every block is selected, and closed forms of attention (q = 0, constant K,
  first prefill token, hand-worked logits in tests/golden/attention_worked_examples.json).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_scores_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BLOCK = 128


# ----------------------------------------------------------------------------- decoders
def test_bf16_decoder_matches_torch_on_every_code():
    codes = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decoder_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert nan.sum() == 2  # 0x7F and 0xFF only: the fn variant has no infinities
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e2m1_decoder_matches_ml_dtypes_on_every_code():
    import ml_dtypes
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle.e2m1_value(int(c)) for c in codes])
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))   # -0.0 for code 8


def test_ue8m0_decoder_matches_torch_and_ml_dtypes_on_every_code():
    import ml_dtypes
    codes = np.arange(256, dtype=np.uint8)
    ref_t = torch.from_numpy(codes.copy()).view(torch.float8_e8m0fnu).double().numpy()
    ref_m = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle.ue8m0_value(int(c)) for c in codes])
    for ref in (ref_t, ref_m):
        nan = np.isnan(ref)
        assert nan.sum() == 1 and nan[255]
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan], ref[~nan])


# ----------------------------------------------------------------------------- helpers
def _small(name, **kw):
    base = wl.WORKLOADS[name]
    return wl.generate(base.scaled(**kw), seed=wl.SEEDS[name] + 100)


def _dense_rows(cache, table_row, L, head):
    """Positions 0..L-1 of one sequence gathered from the paged cache, as fp64 (numpy)."""
    x = cache[table_row[: (L + BLOCK - 1) // BLOCK].long(), head].double()   # [nb,128,128]
    return x.reshape(-1, x.shape[-1])[:L].numpy()


def _positions(ids_row, count, p):
    pos = []
    for j in ids_row[:count]:
        pos.extend(x for x in range(int(j) * BLOCK, int(j) * BLOCK + BLOCK) if x <= p)
    return pos


SCORE_CASES = [
    ("tiny_decode", {}),
    ("spec_decode", dict(batch=3, kv_len=(700, 1500))),
    ("ragged_prefill", dict(batch=2, q_len=(150, 300), prior_len=(0, 400))),
    ("bf16_decode", dict(batch=2, kv_len=(300, 900), H_idxk=8)),
]


# ----------------------------------------------------------------------------- scores
@pytest.mark.parametrize("name,kw", SCORE_CASES)
def test_scores_equal_numpy_brute_force(name, kw):
    p = _small(name, **kw)
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    for b in range(p["batch"]):
        L = p["kv_lens"][b]
        for g in range(p["H_kv"]):
            K = _dense_rows(p["k_idx"], p["table"][b], L, g % p["H_idxk"])     # [L,128]
            Q = p["q_idx"][ro[b]:ro[b + 1], g].double().numpy()               # [q_len,128]
            dots = Q @ K.T                                                    # [q_len, L]
            nbl = p["max_blocks"]
            full = np.full((Q.shape[0], nbl * BLOCK), -np.inf)
            full[:, :L] = dots
            pos_q = cl[b] + np.arange(Q.shape[0])
            full[np.arange(nbl * BLOCK)[None, :] > pos_q[:, None]] = -np.inf
            ref = full.reshape(Q.shape[0], nbl, BLOCK).max(axis=2)
            got = sc[ro[b]:ro[b + 1], g]
            assert np.array_equal(np.isinf(got), np.isinf(ref))
            fin = np.isfinite(ref)
            np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-12, atol=1e-11)


def _dequantized_index_k(p):
    """The scaled index-K cache of ``p`` as fp64 values, decoded with library routines (torch
    for e4m3 and e8m0, ml_dtypes for e2m1): [num_pages, H_idxk, 128, 128]."""
    import ml_dtypes
    codes = p["k_idx"].numpy()
    if p["idx_dtype"] == "fp8":
        v = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
        return v * p["k_idx_scale"].double().numpy()[..., None]
    lo = (codes & 15).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (codes >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    v = np.stack([lo, hi], axis=-1).reshape(codes.shape[:3] + (128,))
    ex = torch.from_numpy(p["k_idx_scale"].numpy().copy()).view(torch.float8_e8m0fnu)
    return v * np.repeat(ex.double().numpy(), 32, axis=-1)


@pytest.mark.parametrize("idx_dtype", ["fp8", "fp4"])
@pytest.mark.parametrize("name,kw", SCORE_CASES)
def test_scaled_index_k_scores_equal_numpy_brute_force(name, kw, idx_dtype):
    p = _small(name, idx_dtype=idx_dtype, **kw)
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"], p["k_idx_scale"], idx_dtype)
    kv = torch.from_numpy(_dequantized_index_k(p))
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    for b in range(p["batch"]):
        L = p["kv_lens"][b]
        for g in range(p["H_kv"]):
            K = _dense_rows(kv, p["table"][b], L, g % p["H_idxk"])
            Q = p["q_idx"][ro[b]:ro[b + 1], g].double().numpy()
            full = np.full((Q.shape[0], p["max_blocks"] * BLOCK), -np.inf)
            full[:, :L] = Q @ K.T
            pos_q = cl[b] + np.arange(Q.shape[0])
            full[np.arange(full.shape[1])[None, :] > pos_q[:, None]] = -np.inf
            ref = full.reshape(Q.shape[0], p["max_blocks"], BLOCK).max(axis=2)
            got = sc[ro[b]:ro[b + 1], g]
            assert np.array_equal(np.isinf(got), np.isinf(ref))
            assert not np.isnan(got).any()
            fin = np.isfinite(ref)
            np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-12, atol=1e-11)


@pytest.mark.parametrize("idx_dtype", ["fp8", "fp4"])
def test_scaled_index_k_is_close_to_the_bf16_cache_it_quantises(idx_dtype):
    """The quantised cache keeps the scores within the formats' rounding (fp8: 2^-4 relative
    per element, fp4: a quarter of the group's scale), and a poisoned token reads as NaN."""
    p16 = _small("bf16_decode", batch=2, kv_len=(300, 900))
    pq = _small("bf16_decode", batch=2, kv_len=(300, 900), idx_dtype=idx_dtype)
    s16 = oracle.index_scores(p16["row_off"], p16["cache_len"], p16["table"], p16["q_idx"],
                              p16["k_idx"], p16["max_blocks"])
    sq = oracle.index_scores(pq["row_off"], pq["cache_len"], pq["table"], pq["q_idx"],
                             pq["k_idx"], pq["max_blocks"], pq["k_idx_scale"], idx_dtype)
    fin = np.isfinite(s16)
    rel = 2.0 ** -4 if idx_dtype == "fp8" else 0.5
    qn = np.linalg.norm(p16["q_idx"].double().numpy(), axis=-1)[..., None]
    assert np.all(np.abs(sq[fin] - s16[fin]) <= rel * np.broadcast_to(qn, s16.shape)[fin] * 12)
    # every pool page beyond the used ones is poisoned through its scale
    assert torch.isnan(pq["k_idx_scale"].float()).any() if idx_dtype == "fp8" else \
        bool((pq["k_idx_scale"] == 0xFF).any())


def test_block_score_is_max_not_mean():
    """A single planted key aligned with q_idx puts its block in the selection even though
    every other position of that block is N(0,1) noise (max over the block, not the mean)."""
    p = _small("bf16_decode", batch=1, kv_len=2000)
    b, g, jstar = 0, 3, 6
    qv = p["q_idx"][0, g].float()
    spike = (50.0 * qv / qv.norm()).to(torch.bfloat16)
    page = int(p["table"][b, jstar])
    p["k_idx"][page, 0, 77] = spike
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    expect = float((qv.double() * spike.double()).sum())
    assert sc[0, g, jstar] == pytest.approx(expect, rel=1e-12)
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], sc, top_k=1, init_blocks=1,
                                    local_blocks=1)
    assert jstar in ids[0, g, :cnt[0, g]].tolist()


# ----------------------------------------------------------------------------- selection
def _select_one(scores, p, init, local, top_k):
    sc = np.full((1, 1, len(scores)), -np.inf)
    sc[0, 0, :] = scores
    ids, cnt = oracle.select_blocks(np.array([0, 1]), np.array([p]), sc, top_k, init, local)
    return ids[0, 0, :cnt[0, 0]].tolist(), ids[0, 0]


def test_select_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLDEN, "select_worked_examples.json")))["cases"]
    for c in cases:
        got, padded = _select_one(c["scores"], c["p"], c["init"], c["local"], c["top_k"])
        assert got == c["expected"], c["name"]
        assert all(x == -1 for x in padded[len(got):])


def _brute_force_select(scores, nb, init, local, top_k):
    forced = {j for j in range(nb) if j < init or j >= nb - local}
    cand = [j for j in range(nb) if j not in forced]
    k = min(top_k, len(cand))
    winners = []
    for subset in itertools.combinations(cand, k):
        rest = [j for j in cand if j not in subset]
        # every kept block beats every dropped one: higher score, or equal score and lower id
        if all(scores[a] > scores[r] or (scores[a] == scores[r] and a < r)
               for a in subset for r in rest):
            winners.append(set(subset))
    assert len(winners) == 1
    return sorted(forced | winners[0])


def test_shared_select_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLDEN, "select_shared_worked_examples.json")))["cases"]
    for c in cases:
        n = c["q_len"]
        mb = max(len(r) for r in c["scores"])
        sc = np.full((n, 1, mb), -np.inf)
        for i, r in enumerate(c["scores"]):
            sc[i, 0, :len(r)] = r
        ids, cnt = oracle.select_blocks_shared(np.array([0, n]), np.array([c["cache_len"]]), sc,
                                               c["top_k"], c["init"], c["local"])
        got = [ids[i, 0, :cnt[i, 0]].tolist() for i in range(n)]
        assert got == c["expected"], c["name"]


@pytest.mark.parametrize("seed", range(30))
def test_shared_select_matches_exhaustive_search(seed):
    """The shared part is the exhaustive top-k of the first token's candidates; each token adds
    its own forced blocks; rows after the first are never read."""
    rng = np.random.default_rng(100 + seed)
    q_len = int(rng.integers(1, 9))
    nb0 = int(rng.integers(1, 11))
    cache_len = (nb0 - 1) * BLOCK + int(rng.integers(0, BLOCK))
    init, local, top_k = (int(x) for x in rng.integers(0, 3, size=3))
    top_k += int(rng.integers(0, 3))
    if init + local + top_k == 0:
        top_k = 1
    nb_last = (cache_len + q_len - 1) // BLOCK + 1
    sc = rng.integers(-3, 4, size=(q_len, 1, nb_last)).astype(np.float64)
    ids, cnt = oracle.select_blocks_shared(np.array([0, q_len]), np.array([cache_len]), sc,
                                           top_k, init, local)
    forced0 = {j for j in range(nb0) if j < init or j >= nb0 - local}
    shared = set(_brute_force_select(sc[0, 0], nb0, init, local, top_k)) - forced0
    for i in range(q_len):
        nb = (cache_len + i) // BLOCK + 1
        forced = {j for j in range(nb) if j < init or j >= nb - local}
        assert ids[i, 0, :cnt[i, 0]].tolist() == sorted(forced | shared)
        assert all(x == -1 for x in ids[i, 0, cnt[i, 0]:])
    # rows after the first do not matter
    sc2 = sc.copy()
    sc2[1:] = rng.normal(size=sc2[1:].shape)
    ids2, cnt2 = oracle.select_blocks_shared(np.array([0, q_len]), np.array([cache_len]), sc2,
                                             top_k, init, local)
    assert np.array_equal(ids, ids2) and np.array_equal(cnt, cnt2)


@pytest.mark.parametrize("name,kw", [("spec_decode", dict(batch=3, kv_len=(700, 1500))),
                                     ("spec_decode", dict(batch=4, q_len=(1, 8),
                                                          kv_len=(100, 900))),
                                     ("bf16_decode", dict(batch=3, kv_len=(300, 2000)))])
def test_shared_select_on_generated_problems(name, kw):
    p = _small(name, **kw)
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    ids, cnt = oracle.select_blocks_shared(p["row_off"], p["cache_len"], sc, p["top_k"],
                                           p["init_blocks"], p["local_blocks"])
    own, own_cnt = oracle.select_blocks(p["row_off"], p["cache_len"], sc, p["top_k"],
                                        p["init_blocks"], p["local_blocks"])
    ro = p["row_off"].tolist()
    for b in range(p["batch"]):
        if ro[b + 1] == ro[b]:
            continue
        t0 = ro[b]
        # the first token keeps its ordinary selection
        assert np.array_equal(ids[t0], own[t0]) and np.array_equal(cnt[t0], own_cnt[t0])
        for t in range(t0, ro[b + 1]):
            for g in range(p["H_kv"]):
                sel = ids[t, g, :cnt[t, g]].tolist()
                assert sel == sorted(set(sel)) and len(sel) >= 1
                assert cnt[t, g] <= p["S"]
    if name == "bf16_decode":       # one token per sequence: sharing changes nothing
        assert np.array_equal(ids, own) and np.array_equal(cnt, own_cnt)


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 11))
    init, local, top_k = (int(x) for x in rng.integers(0, 3, size=3))
    top_k += int(rng.integers(0, 3))
    if init + local + top_k == 0:
        top_k = 1
    # integer-valued scores make ties frequent
    scores = rng.integers(-3, 4, size=nb).astype(np.float64)
    p = (nb - 1) * BLOCK + int(rng.integers(0, BLOCK))
    got, _ = _select_one(scores, p, init, local, top_k)
    assert got == _brute_force_select(scores, nb, init, local, top_k)


def _check_selection_invariants(p, sc, ids, cnt):
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    init, local, top_k = p["init_blocks"], p["local_blocks"], p["top_k"]
    for b in range(p["batch"]):
        for i in range(ro[b + 1] - ro[b]):
            t = ro[b] + i
            nb = (cl[b] + i) // BLOCK + 1
            for g in range(p["H_kv"]):
                sel = ids[t, g, :cnt[t, g]].tolist()
                assert len(sel) >= 1                                   # never empty
                assert sel == sorted(set(sel))                         # ascending, unique
                assert all(0 <= j < nb for j in sel)
                assert all(x == -1 for x in ids[t, g, cnt[t, g]:])
                forced = {j for j in range(nb) if j < init or j >= nb - local}
                assert forced <= set(sel)
                cand = [j for j in range(nb) if j not in forced]
                assert len(sel) == len(forced) + min(top_k, len(cand))
                kept = [sc[t, g, j] for j in cand if j in sel]
                dropped = [sc[t, g, j] for j in cand if j not in sel]
                if kept and dropped:
                    assert min(kept) >= max(dropped)


@pytest.mark.parametrize("name,kw", SCORE_CASES)
def test_selection_invariants(name, kw):
    p = _small(name, **kw)
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], sc, p["top_k"],
                                    p["init_blocks"], p["local_blocks"])
    _check_selection_invariants(p, sc, ids, cnt)


@pytest.mark.parametrize("factor", [2.0, 0.5, 4.0])
def test_selection_is_scale_free(factor):
    """Scaling every index query by a positive power of two (exact in bf16) changes no id:
    only the order of the scores is consumed (ferrox-core 'Four rules': no softmax scale)."""
    p = _small("spec_decode", batch=2, kv_len=(2000, 3000))
    args = (p["top_k"], p["init_blocks"], p["local_blocks"])
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], sc, *args)
    q2 = (p["q_idx"].float() * factor).to(torch.bfloat16)
    assert torch.equal(q2.float(), p["q_idx"].float() * factor)
    sc2 = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], q2, p["k_idx"],
                              p["max_blocks"])
    ids2, cnt2 = oracle.select_blocks(p["row_off"], p["cache_len"], sc2, *args)
    assert np.array_equal(ids, ids2) and np.array_equal(cnt, cnt2)


def test_selection_is_per_kv_head():
    """Head g's selection depends on head g's index query only (no cross-head reduction)."""
    p = _small("bf16_decode", batch=2, kv_len=(5000, 8000))
    args = (p["top_k"], p["init_blocks"], p["local_blocks"])
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], sc, *args)
    g = 5
    q2 = p["q_idx"].clone()
    others = [h for h in range(p["H_kv"]) if h != g]
    q2[:, others] = torch.flip(q2[:, others], dims=[2]) * -1
    sc2 = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], q2, p["k_idx"],
                              p["max_blocks"])
    ids2, cnt2 = oracle.select_blocks(p["row_off"], p["cache_len"], sc2, *args)
    assert np.array_equal(ids[:, g], ids2[:, g])
    assert not np.array_equal(ids[:, others], ids2[:, others])


# ----------------------------------------------------------------------------- attention
def _all_blocks(p):
    """Selection with every visible block (top_k >= nb): ids [total_q,H_kv,S] and counts."""
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    S = p["max_blocks"]
    ids = np.full((p["total_q"], p["H_kv"], S), -1, dtype=np.int32)
    cnt = np.zeros((p["total_q"], p["H_kv"]), dtype=np.int32)
    for b in range(p["batch"]):
        for i in range(ro[b + 1] - ro[b]):
            nb = (cl[b] + i) // BLOCK + 1
            ids[ro[b] + i, :, :nb] = np.arange(nb)
            cnt[ro[b] + i] = nb
    return ids, cnt


def _kv_float(t):
    return t.double()


ATTN_CASES = [
    ("tiny_decode", {}),
    ("spec_decode", dict(batch=2, kv_len=(300, 700), G=3)),
    ("ragged_prefill", dict(batch=2, q_len=(130, 260), prior_len=(0, 300), H_kv=2, G=2)),
    ("fp8_long_decode", dict(batch=2, kv_len=(400, 600), H_kv=2)),
]


@pytest.mark.parametrize("name,kw", ATTN_CASES)
def test_attention_with_every_block_equals_dense_causal_sdpa(name, kw):
    p = _small(name, **kw)
    ids, cnt = _all_blocks(p)
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], ids, cnt, p["scale"])
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    G = p["H_q"] // p["H_kv"]
    for b in range(p["batch"]):
        L = p["kv_lens"][b]
        for g in range(p["H_kv"]):
            K = torch.from_numpy(_dense_rows(p["k"], p["table"][b], L, g))
            V = torch.from_numpy(_dense_rows(p["v"], p["table"][b], L, g))
            Q = p["q"][ro[b]:ro[b + 1], g * G:(g + 1) * G].double().transpose(0, 1)
            pos_q = torch.arange(cl[b], cl[b] + Q.shape[1])
            mask = torch.arange(L)[None, :] <= pos_q[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q[None], K[None, None].expand(1, G, L, 128), V[None, None].expand(1, G, L, 128),
                attn_mask=mask[None, None], scale=p["scale"])[0].transpose(0, 1)
            got = out[ro[b]:ro[b + 1], g * G:(g + 1) * G]
            np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


def _oracle_selection(p):
    sc = oracle.index_scores(p["row_off"], p["cache_len"], p["table"], p["q_idx"], p["k_idx"],
                             p["max_blocks"])
    return oracle.select_blocks(p["row_off"], p["cache_len"], sc, p["top_k"], p["init_blocks"],
                                p["local_blocks"])


def _mean_v_over_selection(p, ids, cnt):
    ro, cl = p["row_off"].tolist(), p["cache_len"].tolist()
    G = p["H_q"] // p["H_kv"]
    ref = np.zeros((p["total_q"], p["H_q"], 128))
    for b in range(p["batch"]):
        V_all = {g: _dense_rows(p["v"], p["table"][b], p["kv_lens"][b], g)
                 for g in range(p["H_kv"])}
        for i in range(ro[b + 1] - ro[b]):
            t = ro[b] + i
            for h in range(p["H_q"]):
                pos = _positions(ids[t, h // G], cnt[t, h // G], cl[b] + i)
                ref[t, h] = V_all[h // G][pos].mean(axis=0)
    return ref


@pytest.mark.parametrize("name,kw", ATTN_CASES[1:])
def test_attention_with_zero_query_is_mean_of_selected_values(name, kw):
    p = _small(name, **kw)
    ids, cnt = _oracle_selection(p)
    p["q"] = torch.zeros_like(p["q"])
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], ids, cnt, p["scale"])
    np.testing.assert_allclose(out, _mean_v_over_selection(p, ids, cnt), rtol=1e-10,
                               atol=1e-12)


def test_attention_with_constant_keys_is_mean_of_selected_values():
    p = _small("spec_decode", batch=2, kv_len=(500, 900))
    ids, cnt = _oracle_selection(p)
    row = torch.randn(128, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    p["k"] = row.expand_as(p["k"]).contiguous()
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], ids, cnt, p["scale"])
    np.testing.assert_allclose(out, _mean_v_over_selection(p, ids, cnt), rtol=1e-9, atol=1e-11)


def test_attention_is_a_convex_combination_of_selected_values():
    p = _small("ragged_prefill", batch=1, q_len=200, prior_len=100, H_kv=2, G=2)
    ids, cnt = _oracle_selection(p)
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], ids, cnt, p["scale"])
    cl = p["cache_len"].tolist()
    V = {g: _dense_rows(p["v"], p["table"][0], p["kv_lens"][0], g) for g in range(2)}
    for i in range(0, 200, 7):
        for h in range(4):
            pos = _positions(ids[i, h // 2], cnt[i, h // 2], cl[0] + i)
            lo, hi = V[h // 2][pos].min(axis=0), V[h // 2][pos].max(axis=0)
            assert np.all(out[i, h] >= lo - 1e-12) and np.all(out[i, h] <= hi + 1e-12)


def test_first_prefill_token_attends_only_to_itself():
    p = _small("ragged_prefill", batch=2, q_len=(129, 140), prior_len=0, H_kv=2, G=2)
    ids, cnt = _oracle_selection(p)
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], ids, cnt, p["scale"])
    ro = p["row_off"].tolist()
    for b in range(2):
        page = int(p["table"][b, 0])
        for h in range(4):
            np.testing.assert_array_equal(out[ro[b], h], p["v"][page, h // 2, 0].double().numpy())


def _golden_problem(c):
    L = c["cache_len"] + c["q_len"]
    nb = (L + BLOCK - 1) // BLOCK
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    q = z(c["q_len"], 1, 128)
    q[:, 0, 0] = c["q"]["dim0"]
    k, v = z(nb, 1, BLOCK, 128), z(nb, 1, BLOCK, 128)
    for r in c["k_rows"]:
        k[r["pos"] // BLOCK, 0, r["pos"] % BLOCK, 0] = r["dim0"]
    for r in c["v_rows"]:
        for key in ("dim0", "dim1"):
            if key in r:
                v[r["pos"] // BLOCK, 0, r["pos"] % BLOCK, int(key[3:])] = r[key]
    ids = np.full((c["q_len"], 1, nb), -1, dtype=np.int32)
    cnt = np.zeros((c["q_len"], 1), dtype=np.int32)
    for i in range(c["q_len"]):
        n = (c["cache_len"] + i) // BLOCK + 1
        ids[i, 0, :n] = np.arange(n)
        cnt[i, 0] = n
    table = np.arange(nb, dtype=np.int32)[None]
    out = oracle.attention(np.array([0, c["q_len"]]), np.array([c["cache_len"]]), table, q, k, v,
                           False, ids, cnt, c["scale"])
    return out


def test_attention_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLDEN, "attention_worked_examples.json")))["cases"]
    env = {"e": math.e}
    for c in cases:
        out = _golden_problem(c)
        exp = c.get("expected") or c.get("expected_token0")
        for key, formula in exp.items():
            assert out[0, 0, int(key[3:])] == pytest.approx(eval(formula, env), rel=1e-14), c["name"]


# ----------------------------------------------------------------------------- latent attention
def _latent(batch=3, q_len=(1, 4), swa_len=(100, 700), comp_len=(300, 900), n_entries=48, H=6,
            window=128, seed=3):
    spec = wl.LATENT_DECODE.scaled(batch=batch, q_len=q_len, swa_len=swa_len,
                                   comp_len=comp_len, n_entries=n_entries, H=H, window=window)
    return wl.generate_latent(spec, seed=seed)


def _latent_oracle(p, **over):
    d = dict(p, **over)
    return oracle.latent_attention(d["row_off"], d["q"], d["window"], d["swa_kv"],
                                   d["swa_layer"], d["swa_len"], d["swa_table"], d["comp_kv"],
                                   d["comp_layer"], d["comp_table"], d["comp_idx"], d["sink"],
                                   d["scale"])


def _leaf_row(kv, table, layer, b, pos):
    return kv[int(table[b, pos // BLOCK]), layer, pos % BLOCK].double()


def _latent_rows(p, t):
    """The K = V rows query t reads, gathered from the two leaves by the layouts' own rules."""
    ro = p["row_off"].tolist()
    b = max(i for i in range(p["batch"]) if ro[i] <= t)
    pos = int(p["swa_len"][b]) + (t - ro[b])
    rows = [_leaf_row(p["swa_kv"], p["swa_table"], p["swa_layer"], b, x)
            for x in range(max(0, pos - p["window"] + 1), pos + 1)]
    rows += [_leaf_row(p["comp_kv"], p["comp_table"], p["comp_layer"], b, int(e))
             for e in p["comp_idx"][t].tolist() if e >= 0]
    return torch.stack(rows)


@pytest.mark.parametrize("seed", [3, 4])
def test_latent_attention_equals_sdpa_with_a_sink_key(seed):
    """torch's scaled_dot_product_attention in fp64 over the gathered rows plus one extra key
    of zeros (value zero) whose additive mask bias is the head's sink."""
    p = _latent(seed=seed)
    got = _latent_oracle(p)
    for t in range(p["total_q"]):
        kv = _latent_rows(p, t)                                      # [n, 128]
        n = kv.shape[0]
        k_ext = torch.cat([kv, torch.zeros(1, 128, dtype=torch.float64)])
        q = p["q"][t].double()[:, None, :]                           # [H, 1, 128]
        bias = torch.zeros(p["H"], 1, n + 1, dtype=torch.float64)
        bias[:, 0, n] = p["sink"].double()
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k_ext[None].expand(p["H"], -1, -1), k_ext[None].expand(p["H"], -1, -1),
            attn_mask=bias, scale=p["scale"])[:, 0]
        np.testing.assert_allclose(got[t], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_latent_attention_with_q_zero_is_the_mean_shrunk_by_the_sink():
    p = _latent(seed=5)
    p["q"] = torch.zeros_like(p["q"])
    got = _latent_oracle(p)
    for t in range(p["total_q"]):
        kv = _latent_rows(p, t)
        n = kv.shape[0]
        ref = kv.sum(0)[None, :] / (torch.exp(p["sink"].double())[:, None] + n)
        np.testing.assert_allclose(got[t], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_latent_attention_without_sink_and_window_is_dense_causal_attention():
    """A window longer than every sequence, no compressed entries and a sink of -inf: ordinary
    causal attention over the whole window leaf (K = V)."""
    p = _latent(seed=6, window=100000)
    p["comp_idx"] = torch.full_like(p["comp_idx"], -1)
    p["sink"] = torch.full_like(p["sink"], -float("inf"))
    got = _latent_oracle(p)
    ro = p["row_off"].tolist()
    for b in range(p["batch"]):
        L = int(p["swa_len"][b]) + ro[b + 1] - ro[b]
        kv = torch.stack([_leaf_row(p["swa_kv"], p["swa_table"], p["swa_layer"], b, x)
                          for x in range(L)])
        q = p["q"][ro[b]:ro[b + 1]].double().permute(1, 0, 2)       # [H, n, 128]
        n = q.shape[1]
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, kv[None].expand(p["H"], -1, -1), kv[None].expand(p["H"], -1, -1),
            attn_mask=mask, scale=p["scale"]).permute(1, 0, 2)
        np.testing.assert_allclose(got[ro[b]:ro[b + 1]], ref.numpy(), rtol=1e-11, atol=1e-12)


def test_latent_attention_window_one_is_a_sigmoid_gate():
    p = _latent(seed=7, window=1)
    p["comp_idx"] = torch.full_like(p["comp_idx"], -1)
    got = _latent_oracle(p)
    for t in range(p["total_q"]):
        v = _latent_rows(p, t)[0]                                     # the query's own row
        z = p["scale"] * (p["q"][t].double() @ v)                     # [H]
        gate = 1.0 / (1.0 + torch.exp(p["sink"].double() - z))
        np.testing.assert_allclose(got[t], (gate[:, None] * v[None]).numpy(), rtol=1e-12,
                                   atol=1e-14)


def test_latent_attention_huge_sink_takes_all_the_mass():
    p = _latent(seed=8)
    p["sink"] = torch.full_like(p["sink"], 1e4)
    assert np.abs(_latent_oracle(p)).max() < 1e-100
