"""GPU parity of gdr_mixer_fwd (the recurrence fused with its token-mixer prologue and
epilogue, through the C ABI) against the fp64 mixer oracle (oracle/mixer.py, which runs
the activations, the sequential recurrence oracle and the RMSNorm-SiLU gate)."""
import numpy as np
import pytest
import torch

import oracle
import workload
from oracle import mixer
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu

EPS = 1e-5


def run_gpu(d, S0=None):
    dd = to_dev(d)
    y, ST = gdr.mixer_fwd(dd["q"], dd["k"], dd["v"], dd["xg"], dd["xb"], dd["xw"], dd["z"], dd["weight"],
                          dd["S0"] if S0 is None else S0, mode=d["mode"], layout=d["layout"],
                          b_range=d["b_range"], eps=EPS)
    torch.cuda.synchronize()
    rc = gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert rc == 0, gdr.gdr_status_string(rc)
    return y, ST


def run_oracle(d):
    return mixer.mixer_fwd(d["q"], d["k"], d["v"], d["xg"], d["xb"], d["xw"], d["z"], d["weight"], d["S0"],
                           mode=d["mode"], eps=EPS, b_range=d["b_range"], token_major=d["layout"] == "bthd")


def check(d):
    y, ST = run_gpu(d)
    y_ref, S_ref = run_oracle(d)
    assert_close("y", np64(y), y_ref, "bf16")
    assert_close("S_T", np64(ST), S_ref, "bf16")


@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_modes_layouts(cuda_ok, layout, mode, T):
    d = workload.make_mixer_inputs(2, 3, T, 128, 128, mode=mode, layout=layout, seed=T + 17,
                                   s0_std=0.05)
    check(d)


@pytest.mark.parametrize("mode", ["gdn2", "kda", "bonly"])
def test_expanded_erase_range(cuda_ok, mode):
    d = workload.make_mixer_inputs(2, 2, 150, 128, 128, mode=mode, layout="bthd", seed=3,
                                   s0_std=0.05, b_range=2.0)
    check(d)


def test_without_initial_state(cuda_ok):
    d = workload.make_mixer_inputs(2, 2, 130, 128, 128, mode="gdn2", layout="bthd", seed=4)
    assert d["S0"] is None
    check(d)


@pytest.mark.parametrize("mode", ["gdn2", "gdn"])
@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
def test_strong_decay_exact_path(cuda_ok, mode, layout):
    # g = -softplus(xg) of about -20 per token: every chunk's cumulative decay passes the
    # tensor-core factorisation limit, so the exact per-pair path runs on the raw inputs
    d = workload.make_mixer_inputs(1, 2, 160, 128, 128, mode=mode, layout=layout, seed=6,
                                   xg_shift=20.0, s0_std=0.1)
    check(d)


def test_mixed_decay_channels(cuda_ok):
    d = workload.make_mixer_inputs(2, 2, 192, 128, 128, mode="gdn2", layout="bthd", seed=8, s0_std=0.1)
    xg = d["xg"].clone()
    xg[..., ::2] = 25.0      # g ~ -25: forgets almost everything per token
    xg[..., 1::2] = -8.0     # g ~ -3e-4: barely decays
    d["xg"] = xg
    check(d)


def test_empty_sequence_copies_state(cuda_ok):
    d = workload.make_mixer_inputs(2, 2, 0, 128, 128, layout="bthd", s0_std=0.2)
    y, ST = run_gpu(d)
    assert y.shape == (2, 0, 2, 128)
    assert torch.equal(ST.cpu(), d["S0"])


def test_matches_separate_activation_and_chunk_fwd(cuda_ok):
    # the fused kernel against the plain forward fed with activations formed on the host
    # in fp64 and rounded to the kernel's input types (the oracle's own prologue)
    d = workload.make_mixer_inputs(2, 2, 257, 128, 128, mode="gdn2", layout="bhtd", seed=9, s0_std=0.05)
    a = mixer.prologue(d["q"], d["k"], d["v"], d["xg"], d["xb"], d["xw"], 1.0)
    bf = lambda x: x.to(torch.bfloat16).cuda()
    o, S_plain = gdr.chunk_fwd(bf(a["q"]), bf(a["k"]), bf(a["v"]), a["g"].float().cuda(), bf(a["b"]),
                               bf(a["w"]), d["S0"].cuda(), mode="gdn2")
    y, ST = run_gpu(d)
    assert_close("S_T fused vs plain", np64(ST), np64(S_plain), "bf16")


def test_mixer_workload_full_size(cuda_ok):
    c = workload.MIXER
    d = workload.make_mixer_inputs(c["B"], c["H"], c["T"], c["dk"], c["dv"], mode=c["mode"],
                                   layout=c["layout"], seed=c["seed"], xg_shift=c["xg_shift"],
                                   s0_std=c["s0_std"])
    y, ST = run_gpu(d)
    assert torch.isfinite(y.float()).all() and torch.isfinite(ST).all()
    # every sequence-head; one sequence (its heads, threaded) at a time bounds the host memory
    yr, Sr = [], []
    for b in range(c["B"]):
        one = lambda x: None if x is None else x[b:b + 1].contiguous()
        dh = dict(q=one(d["q"]), k=one(d["k"]), v=one(d["v"]), xg=one(d["xg"]), xb=one(d["xb"]),
                  xw=one(d["xw"]), z=one(d["z"]), weight=d["weight"], S0=one(d["S0"]),
                  mode=d["mode"], layout=d["layout"], b_range=1.0)
        y_ref, S_ref = run_oracle(dh)
        yr.append(y_ref)
        Sr.append(S_ref)
    y_ref, S_ref = np.concatenate(yr), np.concatenate(Sr)
    if d["layout"] == "bthd":   # per-head slices: heads on the second axis
        y_ref, y_np = y_ref.transpose(0, 2, 1, 3), np64(y).transpose(0, 2, 1, 3)
    else:
        y_np = np64(y)
    assert_close("mixer_t4k y", y_np, y_ref, "bf16")
    assert_close("mixer_t4k S_T", np64(ST), S_ref, "bf16")


@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
def test_host_call_pipelined_in_groups_equals_device_call(cuda_ok, layout):
    d = workload.make_mixer_inputs(3, 2, 150, 128, 128, mode="gdn2", layout=layout, seed=9, s0_std=0.05)
    pin = lambda t: None if t is None else t.pin_memory()
    y_h, S_h = gdr.mixer_fwd_host(pin(d["q"]), pin(d["k"]), pin(d["v"]), pin(d["xg"]), pin(d["xb"]),
                                  pin(d["xw"]), pin(d["z"]), d["weight"], pin(d["S0"]), mode="gdn2",
                                  layout=layout, eps=EPS, groups=2)
    torch.cuda.synchronize()
    y_d, S_d = run_gpu(d)
    assert torch.equal(y_h, y_d.cpu()) and torch.equal(S_h, S_d.cpu())
