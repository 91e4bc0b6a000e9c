"""CPU pin of the factorised chunk forward that the tensor-core kernel computes (decay folded
into Kh, Qg, Kb; the state scaled after its update): its numpy fp64 transcription equals the
sequential oracle to rounding in every mode, with ragged tails and cumulative decays up to the
kernel's factorisation limit (|gamma| <= 60 on a chunk)."""
import numpy as np
import pytest
import torch

import chunk_ref
import oracle
import workload


def compare(d, mode, tol):
    args = (d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"])
    o_ref, S_ref = oracle.fwd(*args, mode=mode)
    o, S = chunk_ref.chunk_fwd_factorised(*args, mode=mode)
    for x, r in ((o, o_ref), (S, S_ref)):
        scale = max(1.0, float(np.abs(r).max()))
        assert float(np.abs(x - r).max()) / scale <= tol


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 70, 150])
def test_factorised_chunk_forward_equals_the_recurrence(mode, T):
    d = workload.make_small(1, 2, T, 16, 16, mode=mode, dtype="f32", seed=T + 5, g_scale=0.5, s0_std=0.1)
    compare(d, mode, 1e-10)


def test_factorised_forward_up_to_the_decay_limit():
    # gamma reaches -57.6 at a chunk's end: Kb = k e^-gamma spans e^57, exact in fp64
    d = workload.make_small(1, 1, 128, 16, 16, mode="gdn2", dtype="f32", seed=9, g_scale=0.5, s0_std=0.1)
    d["g"] = torch.full_like(d["g"], -0.9)
    compare(d, "gdn2", 1e-8)
