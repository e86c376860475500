import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")
    # the C-ABI library is built in-tree (no-op when it is up to date)
    from speculative_decoding_04_b200 import build
    build.build()


@pytest.fixture(autouse=True)
def _default_options():
    yield
    import torch
    if torch.cuda.is_available():
        from speculative_decoding_04_b200 import dspark as D
        D.set_option("draft_path", 0)
        D.set_option("draft_tc_min_b", 1)
        D.set_option("verify_cluster", 0)
        D.set_option("draft_pdl", 1)
        D.set_option("draft_fused", 1)
        D.set_option("verify_persistent", 1)
        D.set_option("verify_impl", 0)
        D.set_option("debug_wait_limit", 0)
        D.set_option("debug_unreachable_barrier", 0)
        D.set_option("verify_groups", 0)
        D.set_option("verify_stream_cluster", 0)
        D.set_option("verify_stream_l2hint", 1)
