"""The allocation-free attention entry point (msa_sparse_attn_paged_noalloc).

It exists for callers that cannot hand the library a workspace (a runtime whose device memory
plan is fixed before serving starts, a plugin interface that passes only inputs and outputs):
its scratch is a device array inside the library.  These tests call it through the C ABI and
check it against msa_sparse_attn_paged with a caller-provided workspace: the kernels and the
split-K partitions are the same, so the outputs must be bit-identical, on two calls in a row
(the array keeps the previous call's contents) and after a call of another shape with many
partitions (its partials are still in the array and must never be read).  They also check
that a shape needing more scratch than the array holds, and a NULL output, are refused before
anything runs.  This file is collected last on purpose.
"""
import pytest
import torch

from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_decode": wl.BF16_DECODE.scaled(batch=6, kv_len=(2000, 9000)),
    "spec_decode": wl.SPEC_DECODE.scaled(batch=5, q_len=(2, 8), kv_len=(1500, 5000)),
    "fp8_decode": wl.FP8_LONG_DECODE.scaled(batch=4, kv_len=(3000, 12000)),
    "prefill": wl.RAGGED_PREFILL.scaled(batch=2, q_len=(60, 300), prior_len=(0, 2000)),
}


def _noalloc(path, out, num_splits=None):
    p = path.p
    msa.msa_sparse_attn_paged_noalloc(path.rp, p["q"], p["k"], p["v"], path.kv_dtype,
                                      path.block_ids, path.num_selected, p["S"], p["H_q"],
                                      p["H_kv"], path.max_blocks, p["scale"],
                                      path.num_splits if num_splits is None else num_splits,
                                      out, path.dev_err)


def _reference(prob, num_splits=0):
    """Scores, selection and the workspace call's output for ``prob``."""
    path = msa.Path(prob, num_splits=num_splits)
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    return path, path.out.clone()


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_call_twice_in_a_row(name):
    prob = wl.generate(CASES[name], seed=4242, device="cuda")
    path, ref = _reference(prob)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        _noalloc(path, out)
        torch.cuda.synchronize()
        assert int(path.dev_err.item()) == 0
        assert torch.equal(out, ref)


def test_noalloc_leftovers_of_a_larger_call_are_never_read():
    """Many split-K partitions on one shape, then a single partition (the attention kernel
    writes the output itself) and a few partitions on another: each equal to the workspace
    call with the same partition count."""
    first = wl.generate(CASES["bf16_decode"], seed=11, device="cuda")
    second = wl.generate(wl.BF16_DECODE.scaled(batch=3, kv_len=(300, 2500)), seed=12,
                         device="cuda")
    for prob, splits in ((first, 61), (second, 1), (second, 3), (first, 2)):
        path, ref = _reference(prob, num_splits=splits)
        out = torch.full_like(ref, float("nan"))
        _noalloc(path, out, num_splits=splits)
        torch.cuda.synchronize()
        assert int(path.dev_err.item()) == 0
        assert torch.equal(out, ref), splits


def test_noalloc_refuses_a_null_output():
    prob = wl.generate(CASES["bf16_decode"], seed=7, device="cuda")
    path, _ = _reference(prob)
    with pytest.raises(msa.MSAError) as ei:
        _noalloc(path, None)
    assert ei.value.status == msa.MSA_ERR_INVALID_ARG


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    prob = wl.generate(CASES["bf16_decode"], seed=7, device="cuda")
    path = msa.Path(prob)
    p = path.p
    # many partitions -> many split-K partials: far more than the array holds
    big = msa.RaggedPaged(path.rp.input_row_offsets, path.rp.cache_lengths,
                          path.rp.kv_lookup_table, 1, 200000, 1, path.rp.max_pages_per_seq,
                          path.rp.num_pages)
    need = msa.msa_attn_workspace_bytes(big, p["S"], p["H_q"], p["H_kv"], path.max_blocks, 0)
    assert need > 32 << 20
    with pytest.raises(msa.MSAError) as ei:
        msa.msa_sparse_attn_paged_noalloc(big, p["q"], p["k"], p["v"], path.kv_dtype,
                                          path.block_ids, path.num_selected, p["S"], p["H_q"],
                                          p["H_kv"], path.max_blocks, p["scale"], 0, path.out)
    assert ei.value.status == msa.MSA_ERR_UNSUPPORTED
