import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    """GPU tests are skipped, not failed, on a machine without a GPU when the
    caller asked for everything; `-m gpu` on a machine with a CUDA device runs them."""
    try:
        import torch

        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


def read_grid(name):
    path = os.path.join(ROOT, "tests", "golden", name)
    rows = [ln.strip() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return rows


def read_numbers(name):
    path = os.path.join(ROOT, "tests", "golden", name)
    vals = {}
    for ln in open(path):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        k, v = [s.strip() for s in ln.split("=")]
        vals[k] = float(v) if "." in v else int(v)
    return vals
