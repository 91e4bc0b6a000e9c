"""GPU parity of gdr_chunk_fwd_split (sequence split into segments) against the oracle
and against the unsplit forward."""
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu


def split_fwd(d, nseg, S0=None, S_T=None):
    return gdr.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"],
                               d["S0"] if S0 is None else S0, mode=d["mode"], nseg=nseg, S_T=S_T)


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("nseg,T", [(2, 200), (3, 640), (5, 1000), (8, 1000), (64, 1000)])
def test_split_matches_oracle(cuda_ok, mode, nseg, T):
    d_cpu = workload.make_small(1, 3, T, 128, 128, mode=mode, dtype="bf16", seed=nseg + T,
                                g_scale=0.1, s0_std=0.05)
    d = to_dev(d_cpu)
    o, ST = split_fwd(d, nseg)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"],
                              d_cpu["w"], d_cpu["S0"], mode=mode)
    assert_close("o", np64(o), o_ref, "bf16")
    assert_close("S_T", np64(ST), S_ref, "bf16")
    # and against the unsplit kernel on the same inputs
    o1, S1 = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode)
    assert_close("o vs unsplit", np64(o), np64(o1), "bf16")


def test_split_strong_decay_and_in_place_state(cuda_ok):
    d_cpu = workload.make_small(2, 2, 700, 128, 128, mode="gdn2", dtype="bf16", seed=3, s0_std=0.1)
    g = d_cpu["g"].clone()
    g[..., ::3] = -4.0             # whole segments forget some channels completely
    d_cpu["g"] = g
    d = to_dev(d_cpu)
    S = d["S0"].clone()
    o, _ = split_fwd(d, 4, S0=S, S_T=S)   # S_T aliases S0
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"],
                              d_cpu["w"], d_cpu["S0"], mode="gdn2")
    assert_close("o", np64(o), o_ref, "bf16")
    assert_close("S_T", np64(S), S_ref, "bf16")


@pytest.mark.parametrize("mode", ["gdn2", "kda"])
def test_split_long_context_workload(cuda_ok, mode):
    wl = workload.CONFIGS["gdn2_t16k"]
    d_cpu = workload.make_inputs(wl, mode=mode)
    d = to_dev(d_cpu)
    nseg = gdr.gdr_chunk_fwd_split_segments(wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.chunk, 1)
    assert nseg > 1
    o, ST = split_fwd(d, nseg)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"],
                              d_cpu["w"], d_cpu["S0"], mode=mode)
    assert_close("o", np64(o), o_ref, "bf16")
    assert_close("S_T", np64(ST), S_ref, "bf16")
