import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def cuda_ok() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_ok():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per checked GPU call: elements more than 1 bf16 ulp from the rounded oracle (near-zero
    outputs included, where the 1-ulp rule is not asserted) and the largest distance."""
    try:
        import gpu_util
    except Exception:
        return
    rows = gpu_util.ULP_RECORDS
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "bf16 ulp distance to bf16(oracle) per checked call")
    tr.write_line(f"{'call':48s} {'elements':>9s} {'>1 ulp':>7s} {'max ulp':>8s} {'err/tol':>8s}")
    for where, n, gt1, mx, et in rows:
        tr.write_line(f"{where[:48]:48s} {n:9d} {gt1:7d} {mx:8d} {et:8.3f}")
    tot = sum(r[1] for r in rows)
    tr.write_line(f"{'all':48s} {tot:9d} {sum(r[2] for r in rows):7d} "
                  f"{max(r[3] for r in rows):8d} {max(r[4] for r in rows):8.3f}")
