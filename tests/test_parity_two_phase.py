"""GPU parity of the two-phase forward (gdr_chunk_fwd_two_phase: the WY records of every
chunk in parallel, then the recurrence over them) against the oracle, on every head, and
against the fused kernel on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu

MODES = ["gdn2", "kda", "gdn", "bonly", "wonly"]


def two_phase(d, nseg, S0=None, S_T=None, workspace=None):
    return gdr.chunk_fwd_two_phase(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"],
                                   d["S0"] if S0 is None else S0, mode=d["mode"], nseg=nseg, S_T=S_T,
                                   workspace=workspace)


def check(d_cpu, o, ST, mode, tag=""):
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"], d_cpu["w"],
                              d_cpu["S0"], mode=mode)
    assert_close("o" + tag, np64(o), o_ref, "bf16")
    assert_close("S_T" + tag, np64(ST), S_ref, "bf16")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("T", [1, 64, 200, 1000])
def test_two_phase_matches_oracle(cuda_ok, mode, T):
    d_cpu = workload.make_small(1, 3, T, 128, 128, mode=mode, dtype="bf16", seed=70 + T, g_scale=0.1,
                                s0_std=0.05)
    d = to_dev(d_cpu)
    o, ST = two_phase(d, 1)
    check(d_cpu, o, ST, mode)
    o1, S1 = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode)
    assert_close("o vs fused", np64(o), np64(o1), "bf16")
    assert_close("S_T vs fused", np64(ST), np64(S1), "bf16")


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn"])
@pytest.mark.parametrize("nseg,T", [(2, 200), (3, 640), (5, 1000), (16, 1000)])
def test_two_phase_split_matches_oracle(cuda_ok, mode, nseg, T):
    d_cpu = workload.make_small(2, 2, T, 128, 128, mode=mode, dtype="bf16", seed=nseg * 7 + T, g_scale=0.1,
                                s0_std=0.05)
    d = to_dev(d_cpu)
    o, ST = two_phase(d, nseg)
    check(d_cpu, o, ST, mode)


@pytest.mark.parametrize("mode", ["gdn2", "gdn", "wonly"])
def test_two_phase_strong_decay_exact_chunks(cuda_ok, mode):
    # channels (or, for the scalar decay, stretches of tokens) decaying fast enough that
    # their chunks leave the factorised path: those chunks' records come from the exact
    # kernel, the rest from the tensor-core one, in one call
    d_cpu = workload.make_small(2, 2, 700, 128, 128, mode=mode, dtype="bf16", seed=5, s0_std=0.1)
    g = d_cpu["g"].clone()
    if mode == "gdn":
        g[:, :, 130:260] = -3.0
        g[0, 1, 500:] = -20.0
    else:
        g[..., ::3] = -4.0
        g[1, 0, :200] = -0.01
    d_cpu["g"] = g
    d = to_dev(d_cpu)
    for nseg in (1, 4):
        o, ST = two_phase(d, nseg)
        check(d_cpu, o, ST, mode, f" nseg={nseg}")


def test_two_phase_every_chunk_exact(cuda_ok):
    d_cpu = workload.make_small(1, 2, 300, 128, 128, mode="kda", dtype="bf16", seed=8, s0_std=0.1,
                                g_const=-2.5)
    d = to_dev(d_cpu)
    o, ST = two_phase(d, 1)
    check(d_cpu, o, ST, "kda")


def test_two_phase_state_in_place_and_zero_start(cuda_ok):
    d_cpu = workload.make_small(1, 4, 333, 128, 128, mode="gdn2", dtype="bf16", seed=9, g_scale=0.2,
                                s0_std=0.1)
    d = to_dev(d_cpu)
    S = d["S0"].clone()
    o, _ = two_phase(d, 3, S0=S, S_T=S)   # S_T aliases S0
    check(d_cpu, o, S, "gdn2", " in place")
    d_cpu["S0"] = None
    d["S0"] = None
    o, ST = two_phase(d, 2)
    check(d_cpu, o, ST, "gdn2", " S0=None")


def test_two_phase_reuses_a_dirty_workspace(cuda_ok):
    # the workspace is scratch: a second call over the first call's leftovers is exact
    d_cpu = workload.make_small(1, 2, 500, 128, 128, mode="gdn2", dtype="bf16", seed=10, g_scale=0.1,
                                s0_std=0.05)
    d = to_dev(d_cpu)
    need = gdr.gdr_chunk_fwd_two_phase_workspace(1, 2, 500, 128, 128, 64, 3)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    o1, S1 = two_phase(d, 3, workspace=ws)
    o2, S2 = two_phase(d, 3, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    check(d_cpu, o2, S2, "gdn2")


@pytest.mark.parametrize("name,mode", [("gdn_t2k", "gdn"), ("gdn2_t16k", "gdn2"), ("gdn2_t16k", "kda")])
def test_two_phase_workloads_full_size_all_heads(cuda_ok, name, mode):
    wl = workload.CONFIGS[name]
    # the planner's segment count where it takes the two-phase path (T = 16K), else one
    nseg = max(1, gdr.gdr_chunk_fwd_two_phase_segments(wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.chunk, 1))
    d_cpu = workload.make_inputs(wl, mode=mode)
    d = to_dev(d_cpu)
    o, ST = two_phase(d, nseg)
    check(d_cpu, o, ST, mode, f" {name}")


def test_two_phase_argument_errors(cuda_ok):
    d = to_dev(workload.make_small(1, 1, 100, 128, 128, mode="gdn2", dtype="bf16", seed=1))
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdr.GdrError) as e:
        two_phase(d, 1, workspace=small)
    assert e.value.code == -8   # GDR_ERR_WORKSPACE
    with pytest.raises(gdr.GdrError):
        two_phase(d, 0)
    d64 = to_dev(workload.make_small(1, 1, 100, 64, 64, mode="gdn2", dtype="bf16", seed=1))
    with pytest.raises(gdr.GdrError):
        two_phase(d64, 1, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    o = torch.full((1, 1, 100, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdr.GdrError):
        gdr.chunk_fwd_two_phase(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], nseg=1, o=o,
                                workspace=small)
    torch.cuda.synchronize()
    assert torch.isnan(o.float()).all(), "a rejected call launches nothing"
