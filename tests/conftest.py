import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")
    # build the in-tree libraries if stale (no-op when up to date), before the
    # test modules import them
    import __graft_entry__

    __graft_entry__.build()


def cuda_ok():
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False
