import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def pytest_sessionstart(session):
    # compile libep.so (sm_100a) and the C oracle if their sources are newer
    from combine_topk_idx_rank_b200 import build as libbuild
    from oracle import build as oracle_build
    libbuild.build()
    oracle_build.build()
