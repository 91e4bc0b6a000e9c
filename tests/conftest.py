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


@pytest.fixture(autouse=True)
def debug_build_bounds_clean(request):
    """With GDR_DEBUG=1 (the debug library, in-kernel bounds checks), every GPU test ends by
    checking that the debug library is the one loaded and that no bounds check failed."""
    yield
    if os.environ.get("GDR_DEBUG") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import linear_attention_recurrence_wy_b200 as gdr
    assert gdr.gdr_debug_build() == 1
    rc = gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert rc != -10, f"bounds check failed at site {gdr.gdr_debug_bounds_site()}"


WORKLOAD_TESTS = ("full_size", "all_heads", "1000_steps", "long_context")


def parity_table(records):
    """Markdown summary of the parity records (util.RECORDS): the measured workloads at full
    size (every sequence-head; a decode run's per-step rows folded into one), then the
    tightest check of each test file, then the totals."""
    def margin(err, worst, tol):
        top = max(err, worst or 0.0)
        return tol / top if top > 0 else float("inf")

    def fmt_row(test, name, what, err, worst, tol):
        m = margin(err, worst, tol)
        w = "" if worst is None else f"{worst:.2e}"
        return f"| {test} | {name} | {what} | {err:.2e} | {w} | {tol:g} | {'exact' if m == float('inf') else f'{m:.1f}x'} |"

    head = ["| test | tensor | metric | whole tensor | worst head | tolerance | margin |",
            "|---|---|---|---|---|---|---|"]
    out = ["## Measured workloads at full size (every sequence-head compared)", ""] + head
    folded = {}
    for test, name, what, err, worst, tol in records:
        if not any(k in test for k in WORKLOAD_TESTS):
            continue
        key = (test, "o (every step)" if name.startswith("o step") else name, what, tol)
        e0, w0, n0 = folded.get(key, (0.0, None, 0))
        folded[key] = (max(e0, err), None if worst is None and w0 is None else max(w0 or 0.0, worst or 0.0), n0 + 1)
    for (test, name, what, tol), (err, worst, n) in folded.items():
        out.append(fmt_row(test.split("::")[-1], name + (f" ({n} checks, max)" if n > 1 else ""), what, err, worst, tol))
    out += ["", "## Tightest check of each test file", ""] + head
    tight = {}
    for r in records:
        f = r[0].split("::")[0]
        if f not in tight or margin(*r[3:]) < margin(*tight[f][3:]):
            tight[f] = r
    for f, r in sorted(tight.items()):
        out.append(fmt_row(r[0].split("/")[-1], *r[1:]))
    out += ["", f"{len(records)} checks in all; tightest margin "
            f"{min(margin(*r[3:]) for r in records):.1f}x of its tolerance."]
    return "\n".join(out) + "\n"


def pytest_sessionfinish(session, exitstatus):
    """With GDR_PARITY_TABLE=<path>, write the achieved parity errors of the session (whole
    tensor, worst sequence-head, tolerance, margin) as a markdown summary."""
    path = os.environ.get("GDR_PARITY_TABLE")
    if not path:
        return
    import util
    if not util.RECORDS:
        return
    with open(path, "w") as f:
        f.write(parity_table(util.RECORDS))
