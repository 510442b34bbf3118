"""msa_decode_step: one call for the whole step, against the separate calls on the same inputs.

On the decode route the attention launch reads each row's scores as soon as the indexer has
published that row's unit (a flag per (sequence, index-K head) tagged with a step counter in
the workspace) instead of waiting for the whole indexer launch; on the other routes the call
runs the stages one after the other.  Either way the scores, the selection and the output are
bit-identical to msa_index_scores_k + msa_select_sparse_attn_paged, call after call, and the
step's counters are left ready for the next call."""
import pytest
import torch

from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl

pytestmark = pytest.mark.gpu

W = wl.WORKLOADS
CASES = {
    "bf16_decode": W["bf16_decode"],
    "bf16_decode_small": W["bf16_decode"].scaled(batch=5, kv_len=(300, 9000)),
    "idxk_per_head": W["bf16_decode"].scaled(batch=3, kv_len=(1000, 5000), H_idxk=8),
    "decode_gqa16": W["bf16_decode"].scaled(batch=3, kv_len=(1500, 6000), H_kv=2, G=16),
    "fp8_decode": W["fp8_long_decode"].scaled(batch=6, kv_len=(2000, 9000)),
    "fp8_index_k": W["fp8_long_decode"].scaled(batch=4, kv_len=(3000, 9000), idx_dtype="fp8"),
    "spec_decode": W["spec_decode"].scaled(batch=4, kv_len=(1500, 5000)),
    "prefill": W["ragged_prefill"].scaled(batch=2, q_len=(50, 200), prior_len=(0, 1500)),
}


def _pair(name, seed=31):
    prob = wl.generate(CASES[name], seed=seed, device="cuda")
    return prob, msa.Path(prob, one_call=True), msa.Path(prob, one_call=False)


@pytest.mark.parametrize("name", sorted(CASES))
def test_one_call_equals_the_separate_calls(name):
    prob, one, two = _pair(name)
    assert one.one_call and not two.one_call
    two.run()
    torch.cuda.synchronize()
    for _ in range(3):  # the step counter moves on every call
        one.out.fill_(0)
        one.run()
        torch.cuda.synchronize()
        assert int(one.dev_err.item()) == 0 and int(two.dev_err.item()) == 0
        assert torch.equal(one.scores, two.scores)
        assert torch.equal(one.num_selected, two.num_selected)
        assert torch.equal(one.block_ids, two.block_ids)
        assert torch.equal(one.out, two.out)


@pytest.mark.parametrize("name", ["bf16_decode_small", "fp8_decode"])
def test_step_counters_are_ready_for_the_next_call(name):
    prob, one, _ = _pair(name)
    words = one.step_workspace[:8].view(torch.int32)
    units = prob["batch"] * prob["max_q_len"] * prob["H_idxk"]
    for k in range(1, 4):
        one.run()
        torch.cuda.synchronize()
        assert int(one.dev_err.item()) == 0
        assert int(words[0].item()) == k        # the step counter
        assert int(words[1].item()) == 0        # the attention's done count
        counters = one.step_workspace[8:8 + 4 * units].view(torch.int32)
        assert int(counters.abs().sum().item()) == 0   # the indexer's per-unit counts
        flags = one.step_workspace[8 + 4 * units:8 + 8 * units].view(torch.int32)
        assert int((flags == k).sum().item()) >= 1     # units published with this step


def test_one_call_refuses_a_workspace_without_room_for_the_flags():
    prob, one, _ = _pair("bf16_decode_small")
    p = prob
    with pytest.raises(msa.MSAError):
        msa.msa_decode_step(one.rp, p["q_idx"], one.kidx, p["top_k"], p["init_blocks"],
                            p["local_blocks"], p["q"], p["k"], p["v"], one.kv_dtype, p["H_q"],
                            p["H_kv"], one.max_blocks, p["scale"], 0, one.step_workspace,
                            one.scores, one.block_ids, one.num_selected, one.out, one.dev_err,
                            workspace_bytes=8)


def test_a_unit_never_published_times_out_and_the_next_call_is_exact():
    """The attention's wait for a unit's flag is bounded.  With the indexer's per-unit counts
    offset so that no CTA of a unit finds itself the last one, no flag goes up: every selecting
    warp gives up after its limit, MSA_DEVERR_TIMEOUT is reported, the launches return (their
    tile loads drained), and once the step's words are zeroed again the next call is exact."""
    import time
    prob, one, two = _pair("bf16_decode_small")
    two.run()
    one.run()
    torch.cuda.synchronize()
    assert int(one.dev_err.item()) == 0
    units = prob["batch"] * prob["max_q_len"] * prob["H_idxk"]
    counters = one.step_workspace[8:8 + 4 * units].view(torch.int32)
    counters.fill_(1 << 20)
    t0 = time.monotonic()
    one.run()
    torch.cuda.synchronize()
    assert time.monotonic() - t0 < 60
    assert int(one.dev_err.item()) & msa.MSA_DEVERR_TIMEOUT
    one.step_workspace[:8 + 8 * units].zero_()
    one.dev_err.zero_()
    one.out.fill_(0)
    one.run()
    torch.cuda.synchronize()
    assert int(one.dev_err.item()) == 0
    assert torch.equal(one.block_ids, two.block_ids)
    assert torch.equal(one.out, two.out)
