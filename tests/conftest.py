import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_sessionstart(session):
    # Rebuild libmsa.so and the oracle when a source is newer than the built library.
    from block_sparse_paged_scores_b200 import build as msa_build
    import oracle
    msa_build.build()
    oracle.build()
