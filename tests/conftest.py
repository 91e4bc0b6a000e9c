import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_sessionfinish(session, exitstatus):
    """With GDR_PARITY_TABLE=<path>, write every achieved parity error of the session
    (whole tensor, worst sequence-head, tolerance, margin) as a markdown table."""
    path = os.environ.get("GDR_PARITY_TABLE")
    if not path:
        return
    import util
    if not util.RECORDS:
        return
    lines = ["| test | tensor | metric | whole tensor | worst head | tolerance | margin |",
             "|---|---|---|---|---|---|---|"]
    for test, name, what, err, worst, tol in util.RECORDS:
        top = max(err, worst or 0.0)
        margin = f"{tol / top:.1f}x" if top > 0 else "exact"
        w = "" if worst is None else f"{worst:.2e}"
        lines.append(f"| {test} | {name} | {what} | {err:.2e} | {w} | {tol:g} | {margin} |")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")
