"""The two-deep host pipeline (msa.HostPipeline): per-step inputs from pinned host memory,
output back to pinned host memory, copies of neighbouring steps overlapped with compute.

Each step's host output must be bit-identical to the same step run on one stream over
device-resident inputs: the pipeline changes where the bytes wait, never what is computed.
Steps differ in their queries so that a buffer handed to the wrong step would show.
"""
import pytest
import torch

from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl

pytestmark = pytest.mark.gpu

W = wl.WORKLOADS
CASES = {
    "bf16_decode": (W["bf16_decode"], dict(batch=4, kv_len=(2000, 9000))),
    "spec_decode": (W["spec_decode"], dict(batch=3, kv_len=(1500, 5000))),
    "fp8_decode": (W["fp8_long_decode"], dict(batch=3, kv_len=(3000, 12000))),
    "prefill": (W["ragged_prefill"], dict(batch=2, q_len=(100, 600), prior_len=(0, 3000))),
}


def _step_inputs(prob, n, seed):
    """n sets of per-step inputs: the problem's own, then fresh queries over the same caches."""
    g = torch.Generator().manual_seed(seed)
    sets = []
    for i in range(n):
        s = {k: prob[k].cpu().clone() for k in msa.HostPipeline.PER_STEP}
        if i:
            for k in ("q", "q_idx"):
                s[k] = (torch.randn(s[k].shape, generator=g) * s[k].float().std()).to(s[k].dtype)
        sets.append({k: v.pin_memory() for k, v in s.items()})
    return sets


@pytest.mark.parametrize("name", sorted(CASES))
def test_pipelined_steps_equal_serial_steps(name):
    spec, kw = CASES[name]
    prob = wl.to_device(wl.generate(spec.scaled(**kw), seed=4242), "cuda")
    steps = _step_inputs(prob, 5, seed=9)

    ref_path = msa.Path(prob)
    expected = []
    for s in steps:
        for k in msa.HostPipeline.PER_STEP:
            prob[k].copy_(s[k])
        ref_path.run()
        expected.append(ref_path.out.cpu())
    torch.cuda.synchronize()
    assert int(ref_path.dev_err.item()) == 0

    pipe = msa.HostPipeline(prob)
    outs = [torch.empty(ref_path.out.shape, dtype=ref_path.out.dtype).pin_memory()
            for _ in steps]
    packed = [pipe.pack(s) for s in steps]
    done = [pipe.submit(s, o) for s, o in zip(packed, outs)]
    pipe.finish(torch.cuda.current_stream())
    torch.cuda.synchronize()
    for p in pipe.paths:
        assert int(p.dev_err.item()) == 0
    assert all(e.query() for e in done[-2:])
    for i, (o, e) in enumerate(zip(outs, expected)):
        assert torch.equal(o, e), f"step {i}"
    # consecutive steps really differed
    assert not torch.equal(expected[0], expected[1])
