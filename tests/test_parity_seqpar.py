"""GPU parity of the sequence split across GPUs: the segment maps and the chaining kernel
(through the C ABI), and three holders emulated one after another on one GPU (their maps
stacked as the all-gather would stack them; the holders' kernels never wait on one
another).  The oracle is the checker: S_local is the oracle's end state from S0, M the
oracle's end state from the identity with v = 0 (so w.v = 0), and the holders' outputs
together the whole-sequence oracle."""
import numpy as np
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, rel_l2, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
from linear_attention_recurrence_wy_b200.seqpar import LibraryOps  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("with_s0", [True, False])
def test_segment_maps_match_oracle(cuda_ok, mode, with_s0):
    d_cpu = workload.make_small(1, 3, 200, 128, 128, mode=mode, dtype="bf16", seed=61, g_scale=0.1,
                                s0_std=0.05 if with_s0 else 0.0)
    d = to_dev(d_cpu)
    S_loc, M = gdr.segment_maps(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode, want_M=True)
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    _, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"], d_cpu["w"], d_cpu["S0"],
                          mode=mode)
    assert_close("S_local", np64(S_loc), S_ref, "bf16")
    eye = torch.eye(128).expand(1, 3, 128, 128).contiguous()
    _, M_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], torch.zeros_like(d_cpu["v"]), d_cpu["g"], d_cpu["b"],
                          d_cpu["w"], eye, mode=mode)
    assert_close("M", np64(M), M_ref, "bf16")
    # without the map: the same end state, and no map
    S2, M2 = gdr.segment_maps(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode)
    torch.cuda.synchronize()
    assert M2 is None and torch.equal(S2, S_loc)


@pytest.mark.parametrize("R", [1, 2, 4])
def test_chain_matches_plain_products(cuda_ok, R):
    gen = torch.Generator().manual_seed(62 + R)
    B, H = 2, 3
    M_all = torch.randn(R, B, H, 128, 128, generator=gen) * 0.08
    S_all = torch.randn(R, B, H, 128, 128, generator=gen)
    S0 = torch.randn(B, H, 128, 128, generator=gen)
    for r in range(R):
        got = gdr.chain_segment_states(M_all.cuda(), S_all.cuda(), S0.cuda() if r == 0 else None, r)
        torch.cuda.synchronize()
        if r == 0:
            ref = S0.double()
        else:
            ref = S_all[0].double()
            for i in range(1, r):
                ref = M_all[i].double() @ ref + S_all[i].double()
        assert rel_l2(np64(got), ref.numpy()) < 1e-5, r


@pytest.mark.parametrize("mode", ["gdn2", "kda"])
def test_three_holders_on_one_gpu_match_the_whole_sequence(cuda_ok, mode):
    T, cuts = 640, [0, 200, 450, 640]   # uneven ranges, not chunk-aligned
    d_cpu = workload.make_small(2, 2, T, 128, 128, mode=mode, dtype="bf16", seed=63, g_scale=0.1, s0_std=0.05)
    d = to_dev(d_cpu)
    ops = LibraryOps()
    R = len(cuts) - 1
    sl = lambda x, r: None if x is None else x[:, :, cuts[r]:cuts[r + 1]].contiguous()
    args = lambda r: [sl(d[n], r) for n in ("q", "k", "v", "g", "b", "w")]
    maps = [ops.maps(*args(r), d["S0"] if r == 0 else None, 0 < r < R - 1, mode, 64) for r in range(R)]
    S_all = torch.stack([m[0] for m in maps])
    M_all = torch.stack([m[1] if m[1] is not None else torch.zeros_like(m[0]) for m in maps])
    outs, S_end = [], None
    for r in range(R):
        S_start = ops.chain(M_all, S_all, d["S0"] if r == 0 else None, r)
        o, S_end = ops.fwd(*args(r), S_start, mode, 64)
        outs.append(o)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"], d_cpu["w"],
                              d_cpu["S0"], mode=mode)
    assert_close("o", np64(torch.cat(outs, 2)), o_ref, "bf16")
    assert_close("S_T", np64(S_end), S_ref, "bf16")


def test_segment_maps_reject_other_shapes(cuda_ok):
    d = to_dev(workload.make_small(1, 1, 64, 64, 64, mode="gdn2", dtype="bf16", seed=1))
    with pytest.raises(gdr.GdrError):
        gdr.segment_maps(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], None, mode="gdn2")
