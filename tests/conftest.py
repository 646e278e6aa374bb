import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_collection_finish(session):
    """Start the oracle runs of the selected full-size stack tests in worker
    processes, so that they overlap the GPU tests collected before them."""
    keys = [item.callspec.params["job"] for item in session.items
            if getattr(item, "module", None) is not None and item.module.__name__ == "test_gpu_stack_fullsize"
            and hasattr(item, "callspec")]
    if not keys:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import _oracle_jobs
    _oracle_jobs.start(keys)


def pytest_sessionfinish(session, exitstatus):
    mod = sys.modules.get("_oracle_jobs")
    if mod is not None:
        mod.shutdown()
