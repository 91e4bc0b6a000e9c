"""CPU pins of the factorised chunk backward that the tensor-core kernel computes (the products
with Kh = b.k.e^gamma, Qg = q.e^gamma, Kb = k.e^-gamma, dA = -dR E^T, dP's diagonal kept
apart, the e^gamma_C-scaled dKe): its numpy fp64 transcription (chunk_bwd_ref) equals the
adjoint of the sequential recurrence (the oracle's backward) to rounding, in every mode, with
ragged tails and cumulative decays up to the kernel's factorisation limit (|gamma| <= 60)."""
import numpy as np
import pytest
import torch

import chunk_bwd_ref
import oracle
import workload

NAMES = ("dq", "dk", "dv", "dg", "db", "dw", "dS0")


def case(B, H, T, d, mode, seed, g_scale=0.5):
    x = workload.make_small(B, H, T, d, d, mode=mode, dtype="f32", seed=seed, g_scale=g_scale, s0_std=0.1)
    gen = torch.Generator().manual_seed(seed + 7)
    dO = torch.randn(B, H, T, d, generator=gen, dtype=torch.float64)
    dST = torch.randn(B, H, d, d, generator=gen, dtype=torch.float64)
    return x, dO, dST


def compare(x, dO, dST, mode, tol=1e-9):
    args = (x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"])
    ref = oracle.bwd(*args, dO, dST, mode=mode)
    got = chunk_bwd_ref.chunk_bwd(*args, dO, dST, mode=mode)
    for n in NAMES:
        if ref[n] is None:
            assert got[n] is None, n
            continue
        assert got[n].shape == ref[n].shape, (n, got[n].shape, ref[n].shape)
        scale = max(1.0, float(np.abs(ref[n]).max()))
        err = float(np.abs(got[n] - ref[n]).max()) / scale
        assert err <= tol, f"{mode} {n}: {err:.2e}"


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 70, 150])
def test_factorised_chunk_backward_equals_the_adjoint(mode, T):
    x, dO, dST = case(1, 2, T, 16, mode, seed=T + 3)
    compare(x, dO, dST, mode)


def test_factorised_form_up_to_the_decay_limit():
    # a constant decay of -0.9 per token: gamma reaches -57.6 at a chunk's end, so Kb = k e^-gamma
    # spans e^57; the products stay exact in fp64
    x, dO, dST = case(1, 1, 128, 16, "gdn2", seed=11)
    x["g"] = torch.full_like(x["g"], -0.9)
    compare(x, dO, dST, "gdn2", tol=1e-7)


def test_without_the_diagonal_term_the_gradients_are_wrong():
    # the separated diagonal of dP carries real gradient: dropping it must break dq and dk
    x, dO, dST = case(1, 1, 64, 16, "gdn2", seed=13)
    args = (x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"])
    ref = oracle.bwd(*args, dO, dST, mode="gdn2")
    got = chunk_bwd_ref.chunk_bwd(*args, dO, dST, mode="gdn2", keep_diagonal=False)   # planted mistake
    rel = lambda a, r: float(np.linalg.norm(a - r) / np.linalg.norm(r))
    assert rel(got["dq"], ref["dq"]) > 1e-3 and rel(got["dk"], ref["dk"]) > 1e-3
    assert rel(got["dv"], ref["dv"]) < 1e-9   # dv does not depend on dP
