import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name: str) -> list[tuple[str, list[str]]]:
    """Key/value lines of a fixture under tests/golden (comments skipped)."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.append((key, vals))
    return rows


@pytest.fixture(scope="session")
def golden():
    return read_golden


def pytest_sessionstart(session):
    """Build the oracle (gcc) and libw4a8.so (nvcc, sm_100a) when stale, so a
    fresh checkout tests what its sources say."""
    import oracle
    from w4a8_quantized_gemm_channel_b200 import build as native_build
    oracle.build()
    native_build.build()


def cuda_ok() -> bool:
    import torch
    return torch.cuda.is_available()
