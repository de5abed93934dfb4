import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))
if str(Path(__file__).resolve().parent) not in sys.path:
    sys.path.insert(0, str(Path(__file__).resolve().parent))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running check (full-size workloads)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as oracle_pkg

    return oracle_pkg.get()


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def sdm():
    import sparse_memory_linear_pkm_b200 as pkg

    pkg.native.load()  # fails loudly when the CUDA library is missing
    return pkg


def env_threads() -> int:
    return int(os.environ.get("SDM_ORACLE_THREADS", "0")) or None
