import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case, minutes of CPU oracle time")


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_sessionfinish(session, exitstatus):
    """Write the session's per-config parity errors and oracle times as JSON
    lines when CQL_METRICS_JSONL names a file."""
    path = os.environ.get("CQL_METRICS_JSONL")
    if not path:
        return
    try:
        from tests.gpu_util import METRICS
    except Exception:
        return
    import json
    with open(path, "w") as f:
        for m in METRICS:
            f.write(json.dumps(m) + "\n")
