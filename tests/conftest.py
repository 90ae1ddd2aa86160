import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")


@pytest.fixture(scope="session")
def cuda_device():
    """The CUDA device for GPU tests; a missing GPU is an error, not a skip."""
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test selected but torch.cuda.is_available() is False")
    return torch.device("cuda:0")


def golden_path(name: str) -> str:
    return os.path.join(ROOT, "tests", "golden", name)


def read_golden(name: str) -> dict:
    """Parse a 'key v1 v2 ...' golden file; '#' lines are comments."""
    out = {}
    with open(golden_path(name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out
