"""Shared helpers of the parity tests: device transfer, error metrics, tolerances.

Tolerances (stated for the forward and the decode step):
  fp32 storage:  max |x - x_oracle| <= 1e-4 over all of o and S_T
  bf16 storage:  ||x - x_oracle||_2 / ||x_oracle||_2 <= 2e-2 for o and for S_T, each
"""
import numpy as np
import torch

TOL_F32_MAXABS = 1e-4
TOL_BF16_RELL2 = 2e-2


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


def worst_head(x, ref, metric):
    """Worst per-(sequence, head) error over the two leading axes (reported beside the
    whole-tensor figure the tolerance applies to); None below three dimensions."""
    if x.ndim < 3 or x.size == 0:
        return None
    xs = x.reshape(x.shape[0] * x.shape[1], -1)
    rs = ref.reshape(ref.shape[0] * ref.shape[1], -1)
    return max(metric(a, b) for a, b in zip(xs, rs))


def assert_close(name, x, ref, dtype):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (name, x.shape, ref.shape)
    assert np.all(np.isfinite(x)), f"{name}: non-finite values"
    if dtype in ("f32", torch.float32):
        metric, tol, what = max_abs, TOL_F32_MAXABS, "max abs"
    else:
        metric, tol, what = rel_l2, TOL_BF16_RELL2, "rel L2"
    err = metric(x, ref)
    worst = worst_head(x, ref, metric)
    report = f"{name}: {what} err {err:.3e}" + ("" if worst is None else f" (worst head {worst:.3e})")
    print(report)
    assert err <= tol, f"{report} > {tol}"
    return err


def gpu_fwd(gdr, d, chunk=64, S0=None, return_state=True):
    S0 = d["S0"] if S0 is None else S0
    return gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S0, mode=d["mode"],
                         chunk=chunk, return_state=return_state)
