import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libkda.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session", autouse=True)
def built_library():
    """Rebuild libkda.so if any CUDA source is newer than it (no-op otherwise)."""
    from hybrid_linear_attention_04_b200 import build
    build.build()


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    return torch.device("cuda", 0)


def pytest_sessionfinish(session, exitstatus):
    """Write the parity measures of this session to $KDA_PARITY_REPORT (when set)."""
    mod = sys.modules.get("kda_cases")
    if mod is not None:
        mod.write_report()
