"""Full-size parity: the five workloads at their real sizes, in the launch configuration the
benchmark times (default split-K partitions), generated on the GPU from the same seeds.

The oracle cannot redo a whole step at these sizes, so each test checks
- properties that hold at any size, on every row: no device error, no NaN, the -inf pattern
  of the block scores, the selection rules against the GPU's own fp32 scores (forced blocks
  present, ascending, the right count, every kept candidate >= every dropped one), and
  bit-identical results on a second run of the step;
- the oracle's answer on sampled query rows, each rebuilt as a one-token problem over the same
  pages (parity_tools.single_row_problem): scores within tolerance, ids bit-exact where the
  cut is separated, attention within tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl
from parity_tools import (check_attention, check_scores, check_selection, head_rows_mask,
                          oracle_forward, single_row_problem)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BLOCK = 128


def _visible_blocks(prob):
    ro = prob["row_off"].cpu().numpy()
    cl = prob["cache_len"].cpu().numpy()
    q_lens = np.diff(ro)
    b_of_t = np.repeat(np.arange(prob["batch"]), q_lens)
    i_of_t = np.arange(prob["total_q"]) - ro[b_of_t]
    return (cl[b_of_t] + i_of_t) // BLOCK + 1


def _check_rules_on_gpu_scores(prob, scores, ids, cnt):
    nb = _visible_blocks(prob)                                    # [tq]
    tq, hkv, mb = scores.shape
    j = np.arange(mb)[None, None, :]
    visible = np.broadcast_to(j < nb[:, None, None], scores.shape)
    assert np.array_equal(np.isneginf(scores), ~visible)
    init, local, top_k = prob["init_blocks"], prob["local_blocks"], prob["top_k"]
    forced = visible & ((j < init) | (j >= nb[:, None, None] - local))
    forced = np.broadcast_to(forced, scores.shape)
    cand = visible & ~forced
    sel = np.zeros(scores.shape, dtype=bool)
    S = ids.shape[2]
    valid = np.arange(S)[None, None, :] < cnt[:, :, None]
    assert np.all(ids[~valid] == -1)
    assert np.all(np.diff(np.where(valid, ids, np.iinfo(np.int32).max), axis=2)[valid[:, :, 1:]] > 0)
    ti, gi, si = np.nonzero(valid)
    sel[ti, gi, ids[ti, gi, si]] = True
    assert np.all(sel <= visible)
    assert np.all(forced <= sel)
    n_forced, n_cand = forced.sum(2), cand.sum(2)
    assert np.array_equal(cnt, n_forced + np.minimum(top_k, n_cand))
    kept = np.where(sel & cand, scores, np.inf).min(2)
    dropped = np.where(~sel & cand, scores, -np.inf).max(2)
    assert np.all(kept >= dropped)


@pytest.mark.parametrize("name", ["tiny_decode", "bf16_decode", "spec_decode", "fp8_long_decode",
                                  "ragged_prefill"])
def test_full_size_workload(name):
    spec = wl.WORKLOADS[name]
    prob = wl.generate(spec, seed=wl.SEEDS[name], device="cuda")
    path = msa.Path(prob)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    scores = path.scores.cpu().numpy()
    ids = path.block_ids.cpu().numpy()
    cnt = path.num_selected.cpu().numpy()
    out = path.out.clone()
    assert not torch.isnan(out.float()).any()
    _check_rules_on_gpu_scores(prob, scores, ids, cnt)

    # the first two stages as one msa_index_select call: the same scores and selection
    fused = msa.Path(prob, fused_select=True)
    fused.index_select()
    torch.cuda.synchronize()
    assert int(fused.dev_err.item()) == 0
    assert np.array_equal(fused.scores.cpu().numpy(), scores)
    assert np.array_equal(fused.block_ids.cpu().numpy(), ids)
    assert np.array_equal(fused.num_selected.cpu().numpy(), cnt)
    assert int(fused.counters.abs().sum().item()) == 0
    del fused

    # the last two stages as one msa_select_sparse_attn_paged call: the same selection and output
    inatt = msa.Path(prob, select_in_attention=True)
    inatt.run()
    torch.cuda.synchronize()
    assert int(inatt.dev_err.item()) == 0
    assert np.array_equal(inatt.block_ids.cpu().numpy(), ids)
    assert np.array_equal(inatt.num_selected.cpu().numpy(), cnt)
    assert torch.equal(inatt.out, out)
    del inatt

    # the same step again: every output bit-identical
    for _ in range(3):
        path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    assert np.array_equal(path.scores.cpu().numpy(), scores)
    assert np.array_equal(path.block_ids.cpu().numpy(), ids)
    assert torch.equal(path.out, out)

    # oracle on sampled rows
    rng = np.random.default_rng(wl.SEEDS[name])
    rows = sorted(set(rng.integers(0, prob["total_q"], size=min(6, prob["total_q"])).tolist()
                      + [0, prob["total_q"] - 1]))
    G = prob["H_q"] // prob["H_kv"]
    for t in rows:
        sub = single_row_problem(prob, t)
        sc, oids, ocnt, oout = oracle_forward(sub)
        nbt = sub["max_blocks"]
        check_scores(scores[t:t + 1, :, :nbt], sc, sub, nbt)
        assert np.all(np.isneginf(scores[t, :, nbt:]))
        same = check_selection(ids[t:t + 1], cnt[t:t + 1], oids, ocnt, sc, sub)
        mask = head_rows_mask(same, G)
        check_attention(out[t:t + 1].float().cpu(), oout, prob["kv_fp8"], rows_mask=mask)
        # every head of the row, near-ties included, against the oracle's attention over the
        # GPU's own selection
        gout = oracle.attention(sub["row_off"], sub["cache_len"], sub["table"], sub["q"],
                                sub["k"], sub["v"], sub["kv_fp8"], ids[t:t + 1], cnt[t:t + 1],
                                sub["scale"])
        check_attention(out[t:t + 1].float().cpu(), gout, prob["kv_fp8"])
