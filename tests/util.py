"""Shared helpers of the parity tests: device transfer, error metrics, tolerances.

Tolerances (stated for the forward and the decode step):
  fp32 storage:  max |x - x_oracle| <= 1e-4 over all of o and S_T
  bf16 storage:  ||x - x_oracle||_2 / ||x_oracle||_2 <= 2e-2 for o and for S_T, each, over
                 the whole tensor AND over every (sequence, head) slice on its own, so a
                 kernel that corrupts one head of many cannot hide behind the others

Every check appends its figures to RECORDS; when GDR_PARITY_TABLE names a file, the
session writes them there as a markdown table (tests/conftest.py).
"""
import os

import numpy as np
import torch

TOL_F32_MAXABS = 1e-4
TOL_BF16_RELL2 = 2e-2

# (test id, tensor, metric, whole-tensor error, worst-head error or None, tolerance)
RECORDS = []


def _test_id():
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def record(name, what, err, worst, tol):
    RECORDS.append((_test_id(), name, what, float(err), None if worst is None else float(worst), tol))


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in d.items()}


def np64(x):
    return x.detach().float().cpu().double().numpy()


def rel_l2(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def worst_head(x, ref, metric, head_axes=2):
    """Worst error over the slices indexed by the `head_axes` leading axes (2 for
    [B, H, ...] tensors, 1 for a stack of sampled heads [n, ...]); None when the tensor
    has no axis left below them or is empty."""
    if x.ndim <= head_axes or x.size == 0:
        return None
    n = int(np.prod(x.shape[:head_axes]))
    xs = x.reshape(n, -1)
    rs = ref.reshape(n, -1)
    return max(metric(a, b) for a, b in zip(xs, rs))


def assert_close(name, x, ref, dtype, head_axes=2):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (name, x.shape, ref.shape)
    assert np.all(np.isfinite(x)), f"{name}: non-finite values"
    if dtype in ("f32", torch.float32):
        metric, tol, what = max_abs, TOL_F32_MAXABS, "max abs"
    else:
        metric, tol, what = rel_l2, TOL_BF16_RELL2, "rel L2"
    err = metric(x, ref)
    worst = worst_head(x, ref, metric, head_axes)
    report = f"{name}: {what} err {err:.3e}" + ("" if worst is None else f" (worst head {worst:.3e})")
    print(report)
    record(name, what, err, worst, tol)
    assert err <= tol, f"{report} > {tol}"
    # max abs over the whole tensor already bounds every head; rel L2 does not
    if worst is not None:
        assert worst <= tol, f"{report}: worst head > {tol}"
    return err


def gpu_fwd(gdr, d, chunk=64, S0=None, return_state=True):
    S0 = d["S0"] if S0 is None else S0
    return gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S0, mode=d["mode"],
                         chunk=chunk, return_state=return_state)
