"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Small cases (the oracle finishes each in seconds) span several page tiles, ragged query
lengths, partial last pages (NaN-poisoned past the sequence end), both index-K layouts,
BF16 and FP8 KV, all three attention routes and several split-K counts.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl
from parity_tools import (block_max_logits, check_attention, check_scores, check_selection,
                          fp32_exact, head_rows_mask, lazy_rescale_events, oracle_forward,
                          plant_large_keys)

pytestmark = pytest.mark.gpu

W = wl.WORKLOADS
CASES = {
    "tiny_decode": (W["tiny_decode"], {}),
    "bf16_decode": (W["bf16_decode"], dict(batch=4, kv_len=(2000, 9000))),
    "bf16_decode_idxk_per_head": (W["bf16_decode"], dict(batch=3, kv_len=(1000, 5000), H_idxk=8)),
    "short_contexts": (W["bf16_decode"], dict(batch=6, kv_len=(1, 300))),
    # decode groups off the swapped-operand path (G > 8) and with padding rows (G = 3)
    "decode_gqa16": (W["bf16_decode"], dict(batch=3, kv_len=(1500, 6000), H_kv=2, G=16)),
    "decode_gqa3": (W["bf16_decode"], dict(batch=4, kv_len=(900, 5000), H_kv=3, G=3)),
    "fp8_decode_gqa16": (W["fp8_long_decode"], dict(batch=2, kv_len=(2000, 7000), H_kv=2,
                                                     G=16)),
    "fp8_decode_gqa5": (W["fp8_long_decode"], dict(batch=3, kv_len=(1000, 4000), H_kv=2, G=5)),
    "spec_decode": (W["spec_decode"], dict(batch=6, kv_len=(1500, 5000))),
    "spec_ragged_q": (W["spec_decode"], dict(batch=6, q_len=(2, 8), kv_len=(1000, 4000))),
    "spec_gqa4": (W["spec_decode"], dict(batch=3, G=4, H_kv=4, q_len=(2, 8), kv_len=(900, 3000))),
    "fp8_decode": (W["fp8_long_decode"], dict(batch=4, kv_len=(3000, 12000))),
    "fp8_spec": (W["fp8_long_decode"], dict(batch=3, q_len=(2, 6), kv_len=(2000, 6000))),
    "prefill": (W["ragged_prefill"], dict(batch=3, q_len=(100, 600), prior_len=(0, 3000))),
    "prefill_from_empty": (W["ragged_prefill"], dict(batch=2, q_len=(9, 300), prior_len=0)),
    "prefill_fp8": (W["ragged_prefill"], dict(batch=2, q_len=(50, 300), prior_len=(0, 2000),
                                              kv_dtype="fp8")),
    "prefill_with_empty_rows": (W["ragged_prefill"], dict(batch=4, q_len=(0, 40),
                                                          prior_len=(100, 900))),
    "prefill_gqa4": (W["ragged_prefill"], dict(batch=2, q_len=(40, 200), prior_len=(0, 1500),
                                               H_kv=2, G=4)),
    "prefill_gqa16": (W["ragged_prefill"], dict(batch=2, q_len=(30, 150), prior_len=(100, 1200),
                                                H_kv=1, G=16)),
}


def _problem(name):
    spec, kw = CASES[name]
    return wl.generate(spec.scaled(**kw), seed=1000 + sorted(CASES).index(name))


_cache = {}


def _oracle(name):
    if name not in _cache:
        p = _problem(name)
        _cache[name] = (p, oracle_forward(p))
    return _cache[name]


def _gpu(prob):
    return wl.to_device(prob, "cuda")


@pytest.mark.parametrize("name", sorted(CASES))
def test_index_scores_match_oracle(name):
    p, (sc, _, _, _) = _oracle(name)
    path = msa.Path(_gpu(p))
    path.index_scores()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_scores(path.scores.cpu().numpy(), sc, p, p["max_blocks"])


@pytest.mark.parametrize("name", sorted(CASES))
def test_select_is_bit_exact_on_identical_scores(name):
    p, (sc, _, _, _) = _oracle(name)
    s32 = fp32_exact(sc)
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], s32, p["top_k"],
                                    p["init_blocks"], p["local_blocks"])
    path = msa.Path(_gpu(p))
    path.select(scores=torch.from_numpy(s32.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_matches_oracle_on_oracle_selection(name):
    p, (_, ids, cnt, out) = _oracle(name)
    path = msa.Path(_gpu(p))
    path.attend(block_ids=torch.from_numpy(ids).cuda(), num_selected=torch.from_numpy(cnt).cuda())
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), out, p["kv_fp8"])


@pytest.mark.parametrize("name", sorted(CASES))
def test_whole_path_matches_oracle(name):
    p, (sc, ids, cnt, out) = _oracle(name)
    path = msa.Path(_gpu(p))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    g_ids, g_cnt = path.block_ids.cpu().numpy(), path.num_selected.cpu().numpy()
    same = check_selection(g_ids, g_cnt, ids, cnt, sc, p)
    assert same.mean() > 0.9
    mask = head_rows_mask(same, p["H_q"] // p["H_kv"])
    check_attention(path.out.float().cpu(), out, p["kv_fp8"], rows_mask=mask)
    # every row, near-ties included, against the oracle's attention over the GPU's selection
    # (a valid top-k under the oracle's scores, checked above)
    out_g = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                             p["kv_fp8"], g_ids, g_cnt, p["scale"])
    check_attention(path.out.float().cpu(), out_g, p["kv_fp8"])


@pytest.mark.parametrize("name,splits", [("bf16_decode", n) for n in (1, 2, 3, 7, 19, 148, 700)]
                         + [("spec_ragged_q", n) for n in (1, 5, 148)]
                         + [("fp8_decode", n) for n in (1, 13, 148)]
                         + [("decode_gqa16", n) for n in (1, 5, 148)]
                         + [("fp8_decode_gqa5", n) for n in (1, 13)])
def test_split_k_partitions_agree(name, splits):
    """Any number of split-K partitions gives the oracle's answer, and the partitions agree with
    one another to fp32 reassociation (a couple of bf16 ulps after rounding)."""
    p, (_, ids, cnt, out) = _oracle(name)
    gids, gcnt = torch.from_numpy(ids).cuda(), torch.from_numpy(cnt).cuda()
    path = msa.Path(_gpu(p), num_splits=splits)
    path.attend(block_ids=gids, num_selected=gcnt)
    base = msa.Path(_gpu(p), num_splits=1)
    base.attend(block_ids=gids, num_selected=gcnt)
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), out, p["kv_fp8"])
    ref = base.out.float()
    diff = (path.out.float() - ref).abs()
    assert float(diff.max()) <= 2 * 2 ** -7 * float(ref.abs().max())


@pytest.mark.parametrize("name", ["bf16_decode", "spec_decode", "fp8_spec"])
def test_partials_then_public_combine_equal_the_fused_call(name):
    p, (_, ids, cnt, out) = _oracle(name)
    gids, gcnt = torch.from_numpy(ids).cuda(), torch.from_numpy(cnt).cuda()
    fused = msa.Path(_gpu(p))
    fused.attend(block_ids=gids, num_selected=gcnt)
    split = msa.Path(_gpu(p))
    split.out.fill_(float("nan"))
    split.attend(block_ids=gids, num_selected=gcnt, combine=False)
    torch.cuda.synchronize()
    assert torch.isnan(split.out.float()).all()          # no combine ran
    n, _, _ = split.partials()
    assert n >= 2
    split.combine()
    torch.cuda.synchronize()
    assert torch.equal(split.out, fused.out)


@pytest.mark.parametrize("ns", [1, 5, 40, 77])
def test_splitk_combine_entry_point(ns):
    torch.manual_seed(0)
    tq, hq = 7, 12
    o = torch.randn(ns, tq, hq, 128, device="cuda")
    lse = torch.randn(ns, tq, hq, device="cuda") * 3
    if ns > 1:
        lse[ns // 2] = -float("inf")            # an empty partition weighs nothing
    if ns > 33:
        lse[33, 2, 5] = 60.0                    # a later chunk holds the largest weight
    lse[:, 3, 4] = -float("inf")                # a row no partition saw -> 0
    out = torch.empty(tq, hq, 128, dtype=torch.bfloat16, device="cuda")
    msa.msa_splitk_combine(o, lse, ns, tq, hq, out)
    torch.cuda.synchronize()
    w = torch.softmax(lse.double(), dim=0).nan_to_num(0.0)
    ref = (w[..., None] * o.double()).sum(0)
    got = out.double()
    assert torch.allclose(got, ref, atol=1e-2, rtol=1e-2)
    assert float(got[3, 4].abs().max()) == 0.0
    if ns == 1:
        assert float((got[:3] - o[0, :3].double()).abs().max()) < 1e-2


def test_all_equal_scores_pick_the_lowest_ids():
    p = wl.generate(W["bf16_decode"].scaled(batch=2, kv_len=(3000, 4000)), seed=77)
    p["k_idx"] = torch.zeros_like(p["k_idx"])
    sc, ids, cnt, _ = oracle_forward(p)
    path = msa.Path(_gpu(p))
    path.index_scores()
    path.select()
    torch.cuda.synchronize()
    gpu_sc = path.scores.cpu().numpy()
    assert np.array_equal(np.isneginf(gpu_sc), np.isneginf(sc))
    assert np.all(gpu_sc[~np.isneginf(gpu_sc)] == 0.0)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)


@pytest.mark.parametrize("top_k,init,local", [(0, 1, 1), (3, 0, 0), (0, 0, 2), (500, 1, 2),
                                              (5, 7, 0)])
def test_selection_edge_parameters(top_k, init, local):
    p, (sc, _, _, _) = _oracle("spec_decode")
    p = dict(p, top_k=top_k, init_blocks=init, local_blocks=local, S=top_k + init + local)
    s32 = fp32_exact(sc)
    ids, cnt = oracle.select_blocks(p["row_off"], p["cache_len"], s32, top_k, init, local)
    path = msa.Path(_gpu(p))
    path.select(scores=torch.from_numpy(s32.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    # and attention over that selection
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           False, ids, cnt, p["scale"])
    path.attend()
    torch.cuda.synchronize()
    check_attention(path.out.float().cpu(), out, False)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_index_select_equals_the_two_stages(name):
    p = _gpu(_problem(name))
    two, one = msa.Path(p), msa.Path(p)
    two.index_scores()
    two.select()
    for _ in range(2):  # the counters must come back to zero for the second call
        one.index_select()
    torch.cuda.synchronize()
    assert int(two.dev_err.item()) == 0 and int(one.dev_err.item()) == 0
    assert torch.equal(one.scores, two.scores)
    assert torch.equal(one.num_selected, two.num_selected)
    assert torch.equal(one.block_ids, two.block_ids)
    assert int(one.counters.abs().sum().item()) == 0


@pytest.mark.parametrize("name", sorted(CASES))
def test_select_in_attention_equals_the_two_stages(name):
    """msa_select_sparse_attn_paged (the selection inside the decode attention launch, two
    launches elsewhere) against msa_select_blocks + msa_sparse_attn_paged."""
    p = _gpu(_problem(name))
    two, one = msa.Path(p, select_in_attention=False), msa.Path(p, select_in_attention=True)
    two.run()
    for _ in range(2):
        one.run()
    torch.cuda.synchronize()
    assert int(two.dev_err.item()) == 0 and int(one.dev_err.item()) == 0
    assert torch.equal(one.num_selected, two.num_selected)
    assert torch.equal(one.block_ids, two.block_ids)
    assert torch.equal(one.out, two.out)


@pytest.mark.parametrize("top_k,init,local", [(0, 1, 1), (3, 0, 0), (0, 0, 2), (500, 1, 2),
                                              (5, 7, 0)])
@pytest.mark.parametrize("name,max_blocks", [("bf16_decode", 0), ("fp8_decode", 0),
                                             ("bf16_decode", 700), ("short_contexts", 1100)])
def test_selection_inside_attention_is_bit_exact(name, max_blocks, top_k, init, local):
    """The in-kernel selection (every register-key variant) against the oracle's on the GPU's
    own scores, and the output against the oracle's attention over that selection."""
    p = _gpu(_problem(name))
    p = dict(p, top_k=top_k, init_blocks=init, local_blocks=local, S=top_k + init + local)
    if max_blocks:
        p = _pad_table(p, max_blocks)
    path = msa.Path(p, max_blocks=max_blocks or None, select_in_attention=True)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in p.items()}
    sc = path.scores.cpu().numpy().astype(np.float64)
    ids, cnt = oracle.select_blocks(cpu["row_off"], cpu["cache_len"], sc, top_k, init, local)
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)
    out = oracle.attention(cpu["row_off"], cpu["cache_len"], cpu["table"], cpu["q"], cpu["k"],
                           cpu["v"], p["kv_fp8"], ids, cnt, p["scale"])
    check_attention(path.out.float().cpu(), out, p["kv_fp8"])


def _pad_table(p, max_pages):
    t = p["table"]
    pad = torch.full((t.shape[0], max_pages - t.shape[1]), -1, dtype=t.dtype, device=t.device)
    return dict(p, table=torch.cat([t, pad], 1))


@pytest.mark.parametrize("top_k,init,local", [(0, 1, 1), (3, 0, 0), (0, 0, 2), (500, 1, 2),
                                              (5, 7, 0), (16, 1, 2)])
@pytest.mark.parametrize("name,max_blocks", [("spec_ragged_q", 0), ("bf16_decode", 0),
                                             ("spec_decode", 300), ("bf16_decode", 700),
                                             ("short_contexts", 1100)])
def test_fused_selection_is_bit_exact(name, max_blocks, top_k, init, local):
    """The fused selection against the oracle's, on the GPU's own scores; a wide score row
    (max_blocks 700 / 1100) takes the 32-key and the from-memory key variants."""
    p = _gpu(_problem(name))
    p = dict(p, top_k=top_k, init_blocks=init, local_blocks=local, S=top_k + init + local)
    if max_blocks:
        p = _pad_table(p, max_blocks)
    path = msa.Path(p, max_blocks=max_blocks or None)
    path.index_select()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    sc = path.scores.cpu().numpy().astype(np.float64)
    ids, cnt = oracle.select_blocks(p["row_off"].cpu().numpy(), p["cache_len"].cpu().numpy(), sc,
                                    top_k, init, local)
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)
    assert int(path.counters.abs().sum().item()) == 0


def test_empty_batch_is_a_no_op():
    p = _gpu(_oracle("tiny_decode")[0])
    empty = dict(p, row_off=torch.zeros(2, dtype=torch.int32, device="cuda"), total_q=0)
    empty["batch"] = 1
    path = msa.Path(empty)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0


def test_bad_page_id_is_reported_not_read():
    p = _gpu(_oracle("bf16_decode")[0])
    p["table"] = p["table"].clone()
    p["table"][1, 3] = p["num_pages"] + 5          # outside the pool
    path = msa.Path(p)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) & msa.MSA_DEVERR_PAGE_ID


@pytest.mark.parametrize("kw", [
    # 8192 one-to-three-page units (per-head index-K): most CTAs of the indexer have no page
    # to score, and the fused selection's last-CTA counting runs over thousands of units
    dict(batch=2048, kv_len=(1, 260), H_kv=4, G=1, H_idxk=4, top_k=1, init_blocks=1,
         local_blocks=0),
    dict(batch=2100, kv_len=(1, 300), H_kv=1, G=1, top_k=1, init_blocks=1, local_blocks=0),
])
def test_indexer_for_many_short_sequences(kw):
    spec = W["bf16_decode"].scaled(**kw)
    p = wl.generate(spec, seed=4242, device="cuda")
    path = msa.Path(p)
    path.index_scores()
    path.select()
    fused = msa.Path(p)
    fused.index_select()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0 and int(fused.dev_err.item()) == 0
    assert torch.equal(fused.scores, path.scores)
    assert torch.equal(fused.block_ids, path.block_ids)
    assert torch.equal(fused.num_selected, path.num_selected)
    assert int(fused.counters.abs().sum().item()) == 0
    cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in p.items()}
    sc = oracle.index_scores(cpu["row_off"], cpu["cache_len"], cpu["table"], cpu["q_idx"],
                             cpu["k_idx"], p["max_blocks"])
    check_scores(path.scores.cpu().numpy(), sc, cpu, p["max_blocks"])
    gsc = path.scores.cpu().numpy().astype(np.float64)
    ids, cnt = oracle.select_blocks(cpu["row_off"], cpu["cache_len"], gsc, p["top_k"],
                                    p["init_blocks"], p["local_blocks"])
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)


# ------------------------------------------------------------------ large late logits
# Every fourth block of each sequence has its keys scaled by 16 (exact), so that a row's
# running maximum jumps up by far more than the prefill kernel's lazy-rescale threshold
# (2^8 in the exp2 domain, about 63 in raw q . k at scale 1/sqrt(128)) at a block that comes
# after blocks it has already accumulated: the rescale of the accumulated output must then
# run, with a factor strictly between 0 and 1.  The opposite case (the largest keys first,
# in block 0, which every row selects) is the "early" plant.
PLANTED = {
    "prefill": ("prefill", 16, 2),                   # tcgen05 route: 16-token tiles, 2 groups
    "prefill_gqa4": ("prefill_gqa4", 32, 2),         # tcgen05, 32-token tiles
    "prefill_fp8": ("prefill_fp8", 1, 1),            # FP8 KV prefill (tile kernel)
    "bf16_decode": ("bf16_decode", 1, 1),
    "decode_gqa16": ("decode_gqa16", 1, 1),
    "spec_decode": ("spec_decode", 1, 1),
    "fp8_decode": ("fp8_decode", 1, 1),
    "fp8_spec": ("fp8_spec", 1, 1),
}


@pytest.mark.parametrize("plant", ["late", "early"])
@pytest.mark.parametrize("name", sorted(PLANTED))
def test_large_logits_after_accumulated_blocks(name, plant):
    base, tile_tokens, groups = PLANTED[name]
    p0 = _problem(base)
    p = plant_large_keys(p0, every=4, phase=3) if plant == "late" else \
        plant_large_keys(p0, every=1 << 30, phase=0)
    sc, ids, cnt, out = oracle_forward(p)
    # the inputs do what they are meant to: the running maximum moves up past the threshold
    # after accumulated blocks (late), or never needs to (early: block 0 holds the largest)
    bmax = block_max_logits(_gpu(p), ids, cnt)
    ev = lazy_rescale_events(p, ids, cnt, bmax, tile_tokens, groups)
    if plant == "late":
        assert ev >= 20, ev
    # the oracle's selection, then the whole path
    path = msa.Path(_gpu(p))
    path.attend(block_ids=torch.from_numpy(ids).cuda(), num_selected=torch.from_numpy(cnt).cuda())
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), out, p["kv_fp8"])
    full = msa.Path(_gpu(p))
    full.run()
    torch.cuda.synchronize()
    assert int(full.dev_err.item()) == 0
    g_ids, g_cnt = full.block_ids.cpu().numpy(), full.num_selected.cpu().numpy()
    check_selection(g_ids, g_cnt, ids, cnt, sc, p)
    out_g = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                             p["kv_fp8"], g_ids, g_cnt, p["scale"])
    check_attention(full.out.float().cpu(), out_g, p["kv_fp8"])


# ------------------------------------------------------------------ scaled index-K caches
SCALED = {
    "fp8idx_decode": (W["bf16_decode"], dict(batch=4, kv_len=(2000, 9000), idx_dtype="fp8")),
    "fp4idx_decode": (W["bf16_decode"], dict(batch=4, kv_len=(2000, 9000), idx_dtype="fp4")),
    "fp8idx_spec": (W["spec_decode"], dict(batch=6, kv_len=(1500, 5000), idx_dtype="fp8")),
    "fp4idx_spec_ragged": (W["spec_decode"], dict(batch=6, q_len=(2, 8), kv_len=(1000, 4000),
                                                   idx_dtype="fp4")),
    "fp8idx_per_head": (W["bf16_decode"], dict(batch=3, kv_len=(1000, 5000), H_idxk=8,
                                               idx_dtype="fp8")),
    "fp4idx_per_head": (W["bf16_decode"], dict(batch=3, kv_len=(1000, 5000), H_idxk=8,
                                               idx_dtype="fp4")),
    "fp4idx_short": (W["bf16_decode"], dict(batch=6, kv_len=(1, 300), idx_dtype="fp4")),
    "fp8idx_fp8kv": (W["fp8_long_decode"], dict(batch=3, kv_len=(3000, 12000),
                                                idx_dtype="fp8")),
    "fp4idx_fp8kv": (W["fp8_long_decode"], dict(batch=3, kv_len=(3000, 12000),
                                                idx_dtype="fp4")),
    "fp8idx_prefill": (W["ragged_prefill"], dict(batch=2, q_len=(40, 200), prior_len=(0, 1500),
                                                 idx_dtype="fp8")),
    "fp4idx_prefill": (W["ragged_prefill"], dict(batch=2, q_len=(40, 200), prior_len=(0, 1500),
                                                 idx_dtype="fp4")),
}


def _scaled_problem(name):
    spec, kw = SCALED[name]
    p = wl.generate(spec.scaled(**kw), seed=2000 + sorted(SCALED).index(name))
    if name.endswith("_decode"):
        # a few rows far beyond f16's range (exact powers of two in bf16): the kernel's
        # per-row prescale must keep them finite
        p["q_idx"] = p["q_idx"].clone()
        p["q_idx"][1] = p["q_idx"][1] * 2.0 ** 17
        p["q_idx"][2, :2] = p["q_idx"][2, :2] * 2.0 ** 40
    return p


_scaled_cache = {}


def _scaled_oracle(name):
    if name not in _scaled_cache:
        p = _scaled_problem(name)
        _scaled_cache[name] = (p, oracle_forward(p))
    return _scaled_cache[name]


@pytest.mark.parametrize("name", sorted(SCALED))
def test_scaled_index_k_scores_match_oracle(name):
    p, (sc, _, _, _) = _scaled_oracle(name)
    path = msa.Path(_gpu(p))
    path.index_scores()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_scores(path.scores.cpu().numpy(), sc, p, p["max_blocks"])


@pytest.mark.parametrize("name", sorted(SCALED))
def test_scaled_index_k_fused_selection_is_bit_exact(name):
    """msa_index_select_k: the same scores as msa_index_scores_k, and the oracle's selection
    on those scores, bit for bit."""
    p = _gpu(_scaled_problem(name))
    one, two = msa.Path(p), msa.Path(p)
    for _ in range(2):
        one.index_select()
    two.index_scores()
    torch.cuda.synchronize()
    assert int(one.dev_err.item()) == 0 and int(two.dev_err.item()) == 0
    assert torch.equal(one.scores, two.scores)
    sc = one.scores.cpu().numpy().astype(np.float64)
    ids, cnt = oracle.select_blocks(p["row_off"].cpu(), p["cache_len"].cpu(), sc, p["top_k"],
                                    p["init_blocks"], p["local_blocks"])
    assert np.array_equal(one.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(one.block_ids.cpu().numpy(), ids)
    assert int(one.counters.abs().sum().item()) == 0


@pytest.mark.parametrize("name", sorted(SCALED))
def test_scaled_index_k_whole_path_matches_oracle(name):
    p, (sc, ids, cnt, out) = _scaled_oracle(name)
    path = msa.Path(_gpu(p))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    g_ids, g_cnt = path.block_ids.cpu().numpy(), path.num_selected.cpu().numpy()
    same = check_selection(g_ids, g_cnt, ids, cnt, sc, p)
    assert same.mean() > 0.9
    out_g = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                             p["kv_fp8"], g_ids, g_cnt, p["scale"])
    check_attention(path.out.float().cpu(), out_g, p["kv_fp8"])


@pytest.mark.parametrize("name", ["bf16_decode", "spec_ragged_q", "bf16_decode_idxk_per_head",
                                  "prefill"])
def test_bf16_descriptor_entry_points_equal_the_bf16_ones(name):
    p = _gpu(_problem(name))
    a, b = msa.Path(p), msa.Path(p)
    a.index_scores()
    msa.msa_index_scores_k(b.rp, p["q_idx"], b.kidx, p["H_kv"], b.max_blocks, 0, b.scores,
                           b.dev_err)
    torch.cuda.synchronize()
    assert torch.equal(a.scores, b.scores)


# ------------------------------------------------------------------ top-k shared across drafts
SHARED = {
    "spec_decode": lambda: _problem("spec_decode"),
    "spec_ragged_q": lambda: _problem("spec_ragged_q"),
    "spec_gqa4": lambda: _problem("spec_gqa4"),
    "fp8_spec": lambda: _problem("fp8_spec"),
    "bf16_decode": lambda: _problem("bf16_decode"),
    "short_contexts": lambda: wl.generate(W["spec_decode"].scaled(batch=8, q_len=(1, 8),
                                                                  kv_len=(9, 400)), seed=31),
    "fp4idx_spec": lambda: _scaled_problem("fp4idx_spec_ragged"),
}


@pytest.mark.parametrize("name", sorted(SHARED))
def test_shared_selection_is_bit_exact(name):
    """msa_index_select_k with MSA_SHARE_ACROSS_DRAFTS: the first tokens' scores against the
    oracle's, every token's selection against the oracle's shared selection on the GPU's own
    scores (bit for bit), twice in a row (counters back at zero)."""
    p = SHARED[name]()
    sc, _, _, _ = oracle_forward(p)
    path = msa.Path(_gpu(p), share_selection=True)
    path.scores.fill_(float("nan"))          # rows after the first must not be read
    for _ in range(2):
        path.index_select()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    assert int(path.counters.abs().sum().item()) == 0
    ro = p["row_off"].tolist()
    assert all(ro[b + 1] > ro[b] for b in range(p["batch"]))
    first = ro[:-1]                          # each sequence's first new token
    g_sc = path.scores.cpu().numpy()
    firsts = dict(p, row_off=torch.arange(p["batch"] + 1, dtype=torch.int32),
                  q_idx=p["q_idx"][first], total_q=p["batch"])
    check_scores(g_sc[first], sc[first], firsts, p["max_blocks"])
    ids, cnt = oracle.select_blocks_shared(p["row_off"], p["cache_len"],
                                           g_sc.astype(np.float64), p["top_k"],
                                           p["init_blocks"], p["local_blocks"])
    assert np.array_equal(path.num_selected.cpu().numpy(), cnt)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)


@pytest.mark.parametrize("name", sorted(SHARED))
def test_shared_selection_whole_path_matches_oracle(name):
    p = SHARED[name]()
    path = msa.Path(_gpu(p), share_selection=True)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    g_ids, g_cnt = path.block_ids.cpu().numpy(), path.num_selected.cpu().numpy()
    out = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                           p["kv_fp8"], g_ids, g_cnt, p["scale"])
    check_attention(path.out.float().cpu(), out, p["kv_fp8"])
    # and against the oracle's own whole shared path wherever the first token's cut is clear
    sc, o_ids, o_cnt, o_out = oracle.forward(p, p["top_k"], p["init_blocks"], p["local_blocks"],
                                             p["scale"], p["max_blocks"], share=True)
    same = np.all(g_ids == o_ids, axis=2) & (g_cnt == o_cnt)
    assert same.mean() > 0.9
    mask = head_rows_mask(same, p["H_q"] // p["H_kv"])
    check_attention(path.out.float().cpu(), o_out, p["kv_fp8"], rows_mask=mask)


def test_shared_selection_is_refused_on_the_prefill_route():
    p = _gpu(_problem("prefill"))
    path = msa.Path(p, share_selection=True)
    with pytest.raises(msa.MSAError) as ei:
        path.index_select()
    assert ei.value.status == msa.MSA_ERR_INVALID_ARG


# ------------------------------------------------------------------ speculative indexer routes
# The speculative route scores BF16 index-K on tcgen05 with a page's positions as M and a
# unit's rows as 32 columns when a unit holds more than 16 rows (the cases above: 4 draft
# tokens x 8 index-query heads), on the warp-MMA kernel otherwise.  Here: 16 rows (two drafts x
# 8 heads) and 8 (one index-K head per KV head, up to 8 tokens x 1 head) on the warp-MMA
# kernel, and 24 (three drafts x 8 heads: a quarter of the columns padding) on tcgen05.
SPEC_TC = {
    "two_drafts": dict(batch=5, q_len=2, kv_len=(700, 5000)),
    "idxk_per_head": dict(batch=4, q_len=(2, 8), kv_len=(900, 4000), H_idxk=8),
    "three_drafts": dict(batch=4, q_len=3, kv_len=(300, 3000)),
}


@pytest.mark.parametrize("name", sorted(SPEC_TC))
def test_speculative_indexer_routes_match_oracle(name):
    p = wl.generate(W["spec_decode"].scaled(**SPEC_TC[name]),
                    seed=3100 + sorted(SPEC_TC).index(name))
    sc, ids, cnt, out = oracle_forward(p)
    path = msa.Path(_gpu(p))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_scores(path.scores.cpu().numpy(), sc, p, p["max_blocks"])
    g_ids, g_cnt = path.block_ids.cpu().numpy(), path.num_selected.cpu().numpy()
    same = check_selection(g_ids, g_cnt, ids, cnt, sc, p)
    assert same.mean() > 0.9
    out_g = oracle.attention(p["row_off"], p["cache_len"], p["table"], p["q"], p["k"], p["v"],
                             p["kv_fp8"], g_ids, g_cnt, p["scale"])
    check_attention(path.out.float().cpu(), out_g, p["kv_fp8"])
