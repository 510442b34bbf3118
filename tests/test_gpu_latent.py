"""GPU parity of the latent sparse attention (msa_latent_sparse_attn_paged) against the CPU
oracle on the same seeded inputs: decode, several new tokens per sequence, head counts that do
not fill a 64-head group, every split count agreeing, padded / repeated / out-of-range entries,
and the other layer of the leaves."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl
from parity_tools import check_attention

pytestmark = pytest.mark.gpu

L = wl.LATENT_DECODE
CASES = {
    "decode": L.scaled(batch=4, swa_len=(100, 3000), comp_len=(300, 1500), n_entries=128),
    "decode_short_leaves": L.scaled(batch=5, swa_len=(0, 40), comp_len=(1, 60), n_entries=64,
                                    H=16),
    "multi_token_h12": L.scaled(batch=3, q_len=(1, 4), swa_len=(200, 900), comp_len=(200, 700),
                                n_entries=96, H=12, window=96),
    "prefill_like": L.scaled(batch=2, q_len=(20, 60), swa_len=(0, 400), comp_len=(100, 400),
                             n_entries=40, H=8, window=256),
    "many_heads": L.scaled(batch=2, swa_len=(500, 900), comp_len=(600, 900), n_entries=200,
                           H=160),
    "layer0": L.scaled(batch=3, swa_len=(300, 700), comp_len=(300, 700), n_entries=64,
                       layer=0),
}


def _problem(name):
    return wl.generate_latent(CASES[name], seed=900 + sorted(CASES).index(name))


def _oracle(p):
    return oracle.latent_attention(p["row_off"], p["q"], p["window"], p["swa_kv"],
                                   p["swa_layer"], p["swa_len"], p["swa_table"], p["comp_kv"],
                                   p["comp_layer"], p["comp_table"], p["comp_idx"], p["sink"],
                                   p["scale"])


def _gpu(p):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in p.items()}


@pytest.mark.parametrize("name", sorted(CASES))
def test_latent_attention_matches_oracle(name):
    p = _problem(name)
    ref = _oracle(p)
    path = msa.LatentPath(_gpu(p))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), ref, False)


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 13, 64])
def test_latent_split_counts_agree(splits):
    p = _problem("decode")
    ref = _oracle(p)
    path = msa.LatentPath(_gpu(p), num_splits=splits)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), ref, False)


def test_latent_entries_padded_repeated_and_out_of_range():
    p = _problem("multi_token_h12")
    ci = p["comp_idx"].clone()
    ci[:, 3] = -1                       # padding in the middle
    ci[:, 5] = ci[:, 4]                 # a repeated entry counts twice
    p["comp_idx"] = ci
    ref = _oracle(p)
    path = msa.LatentPath(_gpu(p))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    check_attention(path.out.float().cpu(), ref, False)
    # an entry past the compressed leaf's end is reported and skipped (never read)
    bad = _gpu(p)
    bad["comp_idx"] = bad["comp_idx"].clone()
    bad["comp_idx"][0, 0] = int(p["comp_len"][0]) + 7
    path = msa.LatentPath(bad)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) & msa.MSA_DEVERR_BLOCK_ID
    assert not torch.isnan(path.out.float()).any()


def test_latent_argument_validation():
    p = _gpu(_problem("decode"))
    path = msa.LatentPath(p)
    for kw in (dict(window=0), dict(scale=0.0), dict(num_splits=65)):
        args = dict(window=p["window"], scale=p["scale"], num_splits=path.num_splits)
        args.update(kw)
        with pytest.raises(msa.MSAError):
            msa.msa_latent_sparse_attn_paged(p["row_off"], p["batch"], p["total_q"],
                                             p["max_q_len"], p["q"], p["H"], path.swa,
                                             args["window"], path.comp, p["comp_idx"],
                                             p["n_entries"], p["sink"], args["scale"],
                                             args["num_splits"], path.workspace, path.out)
