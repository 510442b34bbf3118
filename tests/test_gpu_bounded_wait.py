"""The give-up path of the bounded pipeline waits, on the GPU (msa_selftest_bounded_wait).

Every pipelined kernel of the library waits on mbarriers with a time limit, after which it
reports MSA_DEVERR_TIMEOUT, raises its CTA's abort flag and returns.  Here the same wait runs
on barriers that nothing completes: the first waiter must give up after about its limit, the
second must leave early through the abort flag, a wait on a completed phase must return at
once, and the device must take further work afterwards.  Nothing here can hang: every wait is
bounded.
"""
import pytest
import torch

from block_sparse_paged_scores_b200 import msa
from block_sparse_paged_scores_b200 import workload as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_us", [2000, 20000])
def test_a_wait_that_nothing_completes_gives_up_and_reports(limit_us):
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.zeros(5, dtype=torch.int32, device="cuda")
    msa.msa_selftest_bounded_wait(limit_us, dev_err, result)
    torch.cuda.synchronize()
    r = result.cpu().tolist()
    assert int(dev_err.item()) == msa.MSA_DEVERR_TIMEOUT
    assert r[0] == 2 and r[2] == 2          # both waiters gave up
    assert limit_us <= r[1] < 2 * limit_us + 5000  # the first at its own limit
    assert r[3] < 3 * limit_us              # the second before its own (4x) limit: on the flag
    assert r[4] == 1                        # a completed phase is seen at once
    # the context is still usable: a small whole-path step runs clean afterwards
    path = msa.Path(wl.generate(wl.TINY_DECODE, seed=1, device="cuda"))
    path.run()
    torch.cuda.synchronize()
    assert int(path.dev_err.item()) == 0
    assert not torch.isnan(path.out.float()).any()


def test_selftest_argument_validation():
    result = torch.zeros(5, dtype=torch.int32, device="cuda")
    for bad in (0, 1000001):
        with pytest.raises(msa.MSAError):
            msa.msa_selftest_bounded_wait(bad, None, result)
    with pytest.raises(msa.MSAError):
        msa.msa_selftest_bounded_wait(1000, None, None)
