"""CPU pin of the two-phase forward's algebra (Gated DeltaNet-2 Review §3-2.5, "Chunkwise WY
training": the WY factors of a chunk do not depend on the state, and only the state crosses
chunk borders): the records of every chunk formed first (W = T Kh, U = T (w.v), Qg, Kb, P,
e^gamma_C), then the state pass over them, whole or split into segments whose end states and
transition maps are chained, equals the sequential oracle to rounding in every mode, with
ragged tails and segments."""
import numpy as np
import pytest
import torch

import chunk_ref
import oracle
import workload


def compare(d, mode, nseg, tol=1e-10, C=64):
    args = (d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"])
    o_ref, S_ref = oracle.fwd(*args, mode=mode)
    o, S = chunk_ref.chunk_fwd_two_phase(*args, mode=mode, C=C, nseg=nseg)
    for x, r in ((o, o_ref), (S, S_ref)):
        scale = max(1.0, float(np.abs(r).max()))
        assert float(np.abs(x - r).max()) / scale <= tol


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 70, 200])
def test_two_phase_records_then_state_pass(mode, T):
    d = workload.make_small(1, 2, T, 16, 16, mode=mode, dtype="f32", seed=T + 11, g_scale=0.5, s0_std=0.1)
    compare(d, mode, nseg=1, C=32)


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn"])
@pytest.mark.parametrize("nseg", [2, 3, 5])
def test_two_phase_split_state_pass_chains_segments(mode, nseg):
    # eight chunks of 32 tokens, the last ragged: segments of ceil(8 / nseg) whole chunks (two,
    # three and four segments), the last one short
    d = workload.make_small(1, 2, 7 * 32 + 9, 16, 16, mode=mode, dtype="f32", seed=nseg + 3, g_scale=0.5,
                            s0_std=0.1)
    compare(d, mode, nseg=nseg, C=32)


def test_two_phase_split_without_initial_state():
    d = workload.make_small(1, 1, 160, 16, 16, mode="gdn2", dtype="f32", seed=4, g_scale=0.5, s0_std=0.1)
    d["S0"] = None
    compare(d, "gdn2", nseg=4, C=32)


def test_transition_map_is_the_product_of_the_token_transitions():
    # the map run of a segment equals prod_t (I - b_t.k_t ... ) as applied to a state: check
    # S_end(S) = M S + S_local for a random S, on the record form alone
    d = workload.make_small(1, 1, 96, 16, 16, mode="gdn2", dtype="f32", seed=12, g_scale=0.5, s0_std=0.1)
    recs = chunk_ref.chunk_records(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], "gdn2", C=32)[0][0]
    rng = np.random.default_rng(0)
    S = rng.standard_normal((16, 16))
    M = chunk_ref.state_pass(recs, np.eye(16), with_u=False)
    local = chunk_ref.state_pass(recs, np.zeros((16, 16)))
    assert np.abs(chunk_ref.state_pass(recs, S) - (M @ S + local)).max() <= 1e-10


def test_a_dropped_write_term_in_the_map_run_is_caught():
    # planted mistake: the map run keeps U (the write term): the chained result then differs
    # (five chunks in five segments: the inner segments 1-3 chain through their maps)
    d = workload.make_small(1, 1, 160, 16, 16, mode="gdn2", dtype="f32", seed=21, g_scale=0.5, s0_std=0.1)
    args = (d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"])
    o_ref, _ = oracle.fwd(*args, mode="gdn2")
    good = chunk_ref.state_pass
    try:
        chunk_ref.state_pass = lambda recs, S, with_u=True, out=None: good(recs, S, True, out)
        o_bad, _ = chunk_ref.chunk_fwd_two_phase(*args, mode="gdn2", C=32, nseg=5)
    finally:
        chunk_ref.state_pass = good
    assert float(np.abs(o_bad - o_ref).max()) > 1e-3
