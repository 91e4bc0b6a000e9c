"""GPU parity of gdr_chunk_bwd (the chunkwise gate-aware backward, through the C ABI)
against the fp64 adjoint oracle (oracle.bwd).

Tolerances for the gradients: fp32 storage, max |x - x_oracle| <= 1e-4 * max(1, max |x_oracle|)
per tensor (the forward's 1e-4, scaled to the gradient's size: a gradient sums over up to
T tokens and d channels); bf16 storage, relative L2 <= 2e-2 per tensor and per
sequence-head, as for the forward."""
import numpy as np
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, record, rel_l2, to_dev, worst_head

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "db", "dw", "dS0")


def check_grad(name, x, ref, dtype):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (name, x.shape, ref.shape)
    assert np.all(np.isfinite(x)), f"{name}: non-finite values"
    if dtype == "f32":
        scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
        err = float(np.abs(x - ref).max()) / scale if x.size else 0.0
        print(f"{name}: max abs err / scale {err:.3e} (scale {scale:.2e})")
        record(name, "max abs / scale", err, None, 1e-4)
        assert err <= 1e-4, f"{name}: {err:.3e} > 1e-4"
    else:
        err = rel_l2(x, ref)
        worst = worst_head(x, ref, rel_l2)
        print(f"{name}: rel L2 err {err:.3e}" + ("" if worst is None else f" (worst head {worst:.3e})"))
        record(name, "rel L2", err, worst, 2e-2)
        assert err <= 2e-2, f"{name}: {err:.3e} > 2e-2"
        if worst is not None:
            assert worst <= 2e-2, f"{name}: worst head {worst:.3e} > 2e-2"


def make_case(B, H, T, dk, dv, mode, dtype, seed, s0=0.1, dst=True, g_scale=0.5):
    d = workload.make_small(B, H, T, dk, dv, mode=mode, dtype=dtype, seed=seed, g_scale=g_scale, s0_std=s0)
    gen = torch.Generator().manual_seed(seed + 1000)
    dO = torch.randn(B, H, T, dv, generator=gen).to(workload.torch_dtype(dtype))
    dST = torch.randn(B, H, dk, dv, generator=gen) if dst else None
    return d, dO, dST


def run_case(d, dO, dST, dtype):
    dd = to_dev(d)
    out = gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(),
                        None if dST is None else dST.cuda(), mode=d["mode"])
    torch.cuda.synchronize()
    ref = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode=d["mode"])
    for n in NAMES:
        if ref[n] is None:
            assert out[n] is None
            continue
        check_grad(n, np64(out[n]), ref[n], dtype if n not in ("dg", "dS0") else dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [1, 31, 32, 33, 100])
def test_modes_and_ragged_lengths(cuda_ok, dtype, mode, T):
    d, dO, dST = make_case(2, 2, T, 64, 64, mode, dtype, seed=T + 7)
    run_case(d, dO, dST, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 128), (128, 16), (32, 64), (128, 128)])
def test_dims(cuda_ok, dtype, dk, dv):
    d, dO, dST = make_case(1, 2, 70, dk, dv, "gdn2", dtype, seed=dk + 3 * dv)
    run_case(d, dO, dST, dtype)


@pytest.mark.parametrize("mode", ["gdn2", "gdn"])
def test_without_initial_state_or_state_gradient(cuda_ok, mode):
    d, dO, dST = make_case(2, 2, 90, 64, 64, mode, "f32", seed=5, s0=0.0, dst=False)
    assert d["S0"] is None and dST is None
    run_case(d, dO, dST, "f32")


@pytest.mark.parametrize("g_const", [-20.0, 0.0])
def test_extreme_and_zero_decay(cuda_ok, g_const):
    d, dO, dST = make_case(1, 2, 80, 64, 64, "gdn2", "f32", seed=9)
    d["g"] = torch.full_like(d["g"], g_const)
    run_case(d, dO, dST, "f32")


def test_expanded_erase_range(cuda_ok):
    d = workload.make_small(2, 2, 75, 64, 64, mode="gdn2", dtype="f32", seed=13, g_scale=0.5, s0_std=0.1,
                            b_range=2.0)
    gen = torch.Generator().manual_seed(14)
    run_case(d, torch.randn(2, 2, 75, 64, generator=gen), torch.randn(2, 2, 64, 64, generator=gen), "f32")


def test_empty_sequence_copies_state_gradient(cuda_ok):
    d, dO, dST = make_case(2, 2, 0, 64, 64, "gdn2", "f32", seed=1)
    dd = to_dev(d)
    out = gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(), dST.cuda(),
                        mode="gdn2")
    torch.cuda.synchronize()
    assert torch.equal(out["dS0"].cpu(), dST)


def test_gradient_matches_finite_difference_of_the_gpu_forward(cuda_ok):
    # independent of the oracle: a directional derivative of the GPU forward (fp32 path)
    d, dO, dST = make_case(1, 1, 48, 32, 32, "gdn2", "f32", seed=21, s0=0.2)
    dd = to_dev(d)
    out = gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(), dST.cuda(),
                        mode="gdn2")
    gen = torch.Generator().manual_seed(22)
    dirs = {n: torch.randn(dd[n].shape, generator=gen).cuda() for n in ("q", "k", "v", "g", "b", "w")}

    def L(eps):
        x = {n: dd[n] + eps * dirs[n] for n in dirs}
        o, ST = gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], dd["S0"], mode="gdn2", chunk=32)
        return float((o.double() * dO.cuda().double()).sum() + (ST.double() * dST.cuda().double()).sum())

    h = 1e-2
    fd = (L(h) - L(-h)) / (2 * h)
    ad = sum(float((out["d" + n].double() * dirs[n].double()).sum()) for n in dirs)
    assert abs(fd - ad) <= 2e-3 * max(1.0, abs(ad)), (fd, ad)


def test_t4k_workload_all_heads(cuda_ok):
    # the T=4K workload's shape (B=8, H=16, T=4096, d=128, bf16), every sequence-head
    wl = workload.CONFIGS["gdn2_t4k"]
    d = workload.make_inputs(wl)
    gen = torch.Generator().manual_seed(77)
    dO = torch.randn(wl.B, wl.H, wl.T, wl.dv, generator=gen).to(torch.bfloat16)
    dST = torch.randn(wl.B, wl.H, wl.dk, wl.dv, generator=gen) * 0.1
    dd = to_dev(d)
    out = gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(), dST.cuda(),
                        mode="gdn2")
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    for n in NAMES:
        assert torch.isfinite(out[n].float()).all(), n
    # one sequence (its 16 heads, threaded) at a time bounds the fp64 copies' host memory
    refs = {n: [] for n in NAMES}
    for i in range(wl.B):
        one = lambda x: None if x is None else x[i:i + 1]
        r = oracle.bwd(*(one(d[n]) for n in ("q", "k", "v", "g", "b", "w", "S0")), one(dO), one(dST),
                       mode="gdn2")
        for n in NAMES:
            refs[n].append(r[n])
    for n in NAMES:
        check_grad(f"t4k {n}", np64(out[n]), np.concatenate(refs[n]), "bf16")


# ---- the tensor-core shape (bf16, dk = dv = 128): checkpoints, the state gradient and the
#      per-chunk gradients run on tcgen05; 64-token chunks whose cumulative decay passes e^-60
#      are listed for the CUDA-core per-chunk kernel ------------------------------------------
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("T", [20, 64, 96, 150])
def test_tensor_core_state_gradient(cuda_ok, mode, T):
    # T = 20, 96: a last 64-token span with one 32-token chunk; 64: one whole span
    d, dO, dST = make_case(2, 2, T, 128, 128, mode, "bf16", seed=T + 31, g_scale=0.1, s0=0.05)
    run_case(d, dO, dST, "bf16")


@pytest.mark.parametrize("g_const", [-1.5, -4.0])
def test_tensor_core_state_gradient_strong_decay(cuda_ok, g_const):
    # cumulative decays past the forward kernel's factorisation limit (|gamma| > 60 within a
    # 64-token chunk): the exact path's K_end tiles feed the reverse chain unscaled.  (Much
    # stronger decays leave dg as the exact difference of O(1) pair terms, about zero, where
    # a relative error says nothing; the fp32 path's scaled check covers g = -20.)
    d, dO, dST = make_case(1, 2, 140, 128, 128, "gdn2", "bf16", seed=41, s0=0.05)
    d["g"] = torch.full_like(d["g"], g_const)
    run_case(d, dO, dST, "bf16")


def test_tensor_core_state_gradient_without_state_gradient_input(cuda_ok):
    d, dO, dST = make_case(2, 2, 130, 128, 128, "gdn2", "bf16", seed=43, s0=0.0, dst=False)
    run_case(d, dO, dST, "bf16")


def test_tensor_core_backward_mixed_fast_and_exact_chunks(cuda_ok):
    # strong decay in the first two 64-token chunks (CUDA-core kernel, exact pair decays), mild
    # decay in the last two (tensor-core kernel), in one call
    d, dO, dST = make_case(1, 2, 256, 128, 128, "gdn2", "bf16", seed=47, s0=0.05, g_scale=0.1)
    d["g"][:, :, :128] = -2.0
    run_case(d, dO, dST, "bf16")


def test_tensor_core_backward_many_listed_chunks(cuda_ok):
    # every chunk past the factorisation limit: 16 heads x 41 chunks = 656 listed spans, more
    # than the CUDA-core kernel's grid (4 x 148 CTAs), so its CTAs walk the list; two heads
    # are checked against the oracle
    B, H, T = 1, 16, 2600
    d, dO, dST = make_case(B, H, T, 128, 128, "kda", "bf16", seed=53, s0=0.05)
    d["g"] = torch.full_like(d["g"], -2.0)
    dd = to_dev(d)
    out = gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(), dST.cuda(),
                        mode="kda")
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    heads = [0, 15]
    pick = lambda x: None if x is None else x[:, heads]
    ref = oracle.bwd(*(pick(d[n]) for n in ("q", "k", "v", "g", "b", "w", "S0")), pick(dO), pick(dST), mode="kda")
    for n in NAMES:
        if ref[n] is None:
            continue
        check_grad(f"listed {n}", np64(out[n][:, heads]), ref[n], "bf16")
