"""GPU parity of gdr_chunk_fwd (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workload
from util import assert_close, gpu_fwd, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu


def oracle_full(d):
    return oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=d["mode"])


def oracle_by_sequence(d):
    """The oracle over every sequence-head, one sequence (all its heads, threaded) at a time
    to bound the host memory of the fp64 copies; equal to oracle_full."""
    os_, Ss = [], []
    for i in range(d["q"].shape[0]):
        one = lambda x: None if x is None else x[i:i + 1]
        o, S = oracle.fwd(*(one(d[n]) for n in ("q", "k", "v", "g", "b", "w", "S0")), mode=d["mode"])
        os_.append(o)
        Ss.append(S)
    return np.concatenate(os_), np.concatenate(Ss)


def check_case(d_cpu, chunk, dtype):
    d = to_dev(d_cpu)
    o, ST = gpu_fwd(gdr, d, chunk=chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_full(d_cpu)
    e1 = assert_close("o", np64(o), o_ref, dtype)
    e2 = assert_close("S_T", np64(ST), S_ref, dtype)
    return e1, e2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 17, 64, 65, 200])
def test_small_shapes_modes(cuda_ok, dtype, mode, T):
    d = workload.make_small(2, 3, T, 64, 64, mode=mode, dtype=dtype, seed=T, g_scale=0.5,
                            s0_std=0.1)
    check_case(d, 64, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (16, 128), (128, 16)])
def test_dims_and_chunks(cuda_ok, dtype, chunk, dk, dv):
    d = workload.make_small(1, 2, 150, dk, dv, mode="gdn2", dtype=dtype, seed=dk + dv + chunk,
                            g_scale=0.3, s0_std=0.05)
    check_case(d, chunk, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["gdn2", "gdn"])
def test_without_initial_state(cuda_ok, dtype, mode):
    d = workload.make_small(2, 2, 130, 128, 128, mode=mode, dtype=dtype, seed=7, s0_std=0.0)
    assert d["S0"] is None
    check_case(d, 64, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("g_const", [-20.0, -3.0, 0.0])
def test_extreme_and_zero_decay(cuda_ok, dtype, g_const):
    d = workload.make_small(1, 2, 160, 128, 128, mode="gdn2", dtype=dtype, seed=3, s0_std=0.1,
                            g_const=g_const)
    check_case(d, 64, dtype)


@pytest.mark.parametrize("g_scale", [1.0, 1.3])
def test_decay_near_fast_path_limit(cuda_ok, g_scale):
    # cumulative chunk decays of about 50-70 nats: some chunks on either side of the
    # tensor-core kernel's factorisation limit
    d = workload.make_small(2, 4, 256, 128, 128, mode="gdn2", dtype="bf16", seed=5,
                            g_scale=g_scale, s0_std=0.05)
    check_case(d, 64, "bf16")


def test_mixed_extreme_decay_channels(cuda_ok):
    # half the channels forget almost everything per token, half barely decay
    d = workload.make_small(2, 2, 192, 128, 128, mode="gdn2", dtype="bf16", seed=4, s0_std=0.1)
    g = d["g"].clone()
    g[..., ::2] = -25.0
    g[..., 1::2] = -1e-3
    d["g"] = g
    check_case(d, 64, "bf16")


def test_empty_sequence_copies_state(cuda_ok):
    d = to_dev(workload.make_small(2, 2, 0, 64, 64, s0_std=0.2))
    o, ST = gpu_fwd(gdr, d)
    torch.cuda.synchronize()
    assert o.shape == (2, 2, 0, 64)
    assert torch.equal(ST, d["S0"])


def test_in_place_state_and_split_sequence(cuda_ok):
    d_cpu = workload.make_small(2, 2, 200, 128, 128, mode="gdn2", dtype="f32", seed=9, s0_std=0.1)
    d = to_dev(d_cpu)
    o_full, S_full = gpu_fwd(gdr, d)
    cut = 77   # not a multiple of the chunk
    part = lambda x, s: None if x is None else x[:, :, s].contiguous()
    S = d["S0"].clone()
    outs = []
    for sl in (slice(0, cut), slice(cut, None)):
        dd = {k: part(d[k], sl) for k in ("q", "k", "v", "g", "b", "w")}
        o, _ = gdr.chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], S,
                             mode="gdn2", S_T=S)       # S_T aliases S0: in-place update
        outs.append(o)
    torch.cuda.synchronize()
    assert_close("o split", np64(torch.cat(outs, 2)), np64(o_full), "f32")
    assert_close("S split", np64(S), np64(S_full), "f32")


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
def test_decode_steps_equal_chunk_forward(cuda_ok, mode):
    d_cpu = workload.make_small(2, 2, 40, 64, 64, mode=mode, dtype="f32", seed=11, s0_std=0.1)
    d = to_dev(d_cpu)
    o_full, S_full = gpu_fwd(gdr, d, chunk=16)
    S = d["S0"].clone()
    step = lambda x, t: None if x is None else x[:, :, t].contiguous()
    for t in range(40):
        o_t = gdr.decode_step(*(step(d[k], t) for k in ("q", "k", "v", "g", "b", "w")), S, mode=mode)
        assert_close(f"o[{t}]", np64(o_t), np64(o_full[:, :, t]), "f32")
    torch.cuda.synchronize()
    assert_close("S", np64(S), np64(S_full), "f32")


# ---- gate-ablation variants on the tensor-core path (dk = dv = 128, bf16) --------------
@pytest.mark.parametrize("mode,b_range", [("bonly", 1.0), ("wonly", 1.0), ("gdn2", 2.0),
                                          ("bonly", 2.0)])
@pytest.mark.parametrize("T", [65, 200])
def test_variants_tensor_core(cuda_ok, mode, b_range, T):
    """b-only, w-only and the expanded erase range b in [0, 2] (Gated DeltaNet-2 Review,
    gate ablation) through the tcgen05 kernel."""
    d = workload.make_small(2, 2, T, 128, 128, mode=mode, dtype="bf16", seed=T + 3, g_scale=0.1,
                            s0_std=0.05, b_range=b_range)
    check_case(d, 64, "bf16")


# ---- the measured workloads, at full size; every sequence-head vs the oracle -------------
@pytest.mark.parametrize("name,mode", [("gdn2_tiny", "gdn2"), ("gdn_t2k", "gdn"),
                                       ("gdn2_t4k", "gdn2"), ("gdn2_t16k", "gdn2"),
                                       ("gdn2_t16k", "kda")])
def test_workloads_full_size(cuda_ok, name, mode):
    wl = workload.CONFIGS[name]
    d_cpu = workload.make_inputs(wl, mode=mode)
    d = to_dev(d_cpu)
    o, ST = gpu_fwd(gdr, d, chunk=wl.chunk)
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    o_ref, S_ref = oracle_by_sequence(d_cpu)
    assert_close(f"{name} o", np64(o), o_ref, wl.dtype)
    assert_close(f"{name} S_T", np64(ST), S_ref, wl.dtype)


@pytest.mark.parametrize("groups", [1, 4, 7])
def test_host_call_pipelined_in_groups_equals_device_call(cuda_ok, groups):
    # the end-to-end host path splits the sequence-heads into contiguous groups whose copies
    # overlap the computation; per sequence-head the kernel is deterministic, so the result
    # must equal the one-shot device call bit for bit (7 groups of 6 units: some empty)
    d_cpu = workload.make_small(2, 3, 200, 128, 128, mode="gdn2", dtype="bf16", seed=31, g_scale=0.1,
                                s0_std=0.05)
    hin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in d_cpu.items()}
    o_h, S_h = gdr.chunk_fwd_host(hin["q"], hin["k"], hin["v"], hin["g"], hin["b"], hin["w"], hin["S0"],
                                  mode="gdn2", groups=groups)
    torch.cuda.synchronize()
    d = to_dev(d_cpu)
    o_d, S_d = gpu_fwd(gdr, d)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(S_h, S_d.cpu())
