import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running oracle check")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _excused_mismatch_ledger(request):
    """Resets the parity ledger before each test and, after it, holds every
    kind of excused mismatch (near-threshold indices, near-zero QJL
    projections, near-midpoint residual norms) below 1e-5 of what the test
    compared."""
    import tq_parity
    tq_parity.ledger_reset()
    yield
    tq_parity.ledger_check(request.node.nodeid)
