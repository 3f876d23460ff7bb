"""Shared pytest configuration.

Markers:
  gpu  -- needs a CUDA device (B200, sm_100a); run with ``-m gpu``.
Everything unmarked runs on a CPU-only host.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device on this host")
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def lib(cuda_device):
    """The CUDA library through its Python binding.  On a GPU host a missing
    or unloadable library is an error, never a skip."""
    import tensor_allreduce_residual_ar_b200 as ar
    ar.load_library()
    return ar


@pytest.fixture(scope="session")
def parity_report():
    """Collects per-workload error statistics from the GPU parity tests.
    When AR_PARITY_REPORT names a file, the collected lines are written there
    as JSON at the end of the session (nothing is written otherwise)."""
    import json
    rows = []

    def add(name, stats):
        rows.append({"case": name, **{k: v for k, v in stats.items()}})

    yield add
    path = os.environ.get("AR_PARITY_REPORT")
    if path and rows:
        with open(path, "w") as f:
            for r in rows:
                f.write(json.dumps(r) + "\n")


@pytest.fixture(autouse=True)
def _clear_forced_plans(request):
    """A plan forced by one test never leaks into the next: after every test
    that used the library, every variant goes back to the plan table."""
    yield
    if "lib" in request.fixturenames:
        import tensor_allreduce_residual_ar_b200 as ar
        for variant in (0, 1, 2):
            ar.ar_plan_force(variant, 0)
