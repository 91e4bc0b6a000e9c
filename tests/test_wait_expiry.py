"""The expiry path of the kernels' bounded waits, run for real on the GPU.

Every mbarrier wait in the tensor-core forward, the streaming decode kernel and the
tensor-core per-chunk backward is bounded; when a bound runs out, the kernel raises its
abort flag, drains its own bulk copies and tensor-core work, frees its tensor memory and
returns, and gdr_last_device_error() reports GDR_ERR_TIMEOUT.  The test hook
gdr_test_set_first_wait_limit(1) makes the first wait of each CTA give up after one
non-blocking poll, while the producer it waits for (the WY group, or a bulk copy still in
flight) is merely slow -- nothing is made to hang.  Each case then checks that the error
is reported once, that the next normal call matches the oracle and reports no error, so
nothing was left waiting or holding tensor memory."""
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu

TIMEOUT = -7


def stream():
    return torch.cuda.current_stream().cuda_stream


def expire_once(call):
    """Run `call` with the first wait of each CTA bounded to one poll; return the status
    gdr_last_device_error reports afterwards (and check that reading it clears it)."""
    assert gdr.gdr_last_device_error(stream()) == 0
    gdr.gdr_test_set_first_wait_limit(1)
    try:
        call()
        rc = gdr.gdr_last_device_error(stream())
    finally:
        gdr.gdr_test_set_first_wait_limit(0)
    assert gdr.gdr_last_device_error(stream()) == 0   # read and cleared
    return rc


@pytest.mark.parametrize("mode", ["gdn2", "kda"])
def test_forward_first_wait_expires_then_recovers(cuda_ok, mode):
    d_cpu = workload.make_small(2, 4, 640, 128, 128, mode=mode, dtype="bf16", seed=21, g_scale=0.1,
                                s0_std=0.05)
    d = to_dev(d_cpu)
    run = lambda: gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode)
    assert expire_once(run) == TIMEOUT
    o, ST = run()
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(stream()) == 0
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"], d_cpu["w"],
                              d_cpu["S0"], mode=mode)
    assert_close("o after expiry", np64(o), o_ref, "bf16")
    assert_close("S_T after expiry", np64(ST), S_ref, "bf16")


def test_decode_first_wait_expires_then_recovers(cuda_ok):
    # more heads than SMs at d = 128: the streaming kernel, every CTA's first state copy
    N, H, d_ = 64, 16, 128
    dd = workload.make_small(N, H, 1, d_, d_, mode="gdn2", dtype="bf16", seed=22, s0_std=0.2)
    S0 = torch.randn(N, H, d_, d_, generator=torch.Generator().manual_seed(23)) * 0.2
    args = [None if dd[k] is None else dd[k][:, :, 0].contiguous() for k in ("q", "k", "v", "g", "b", "w")]
    dev = [None if x_ is None else x_.cuda() for x_ in args]
    S_bad = S0.cuda()
    assert expire_once(lambda: gdr.decode_step(*dev, S_bad, mode="gdn2")) == TIMEOUT
    S = S0.cuda()
    o = gdr.decode_step(*dev, S, mode="gdn2")
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(stream()) == 0
    o_ref, S_ref = oracle.decode(*args, S=S0, mode="gdn2")
    assert_close("o after expiry", np64(o), o_ref, "bf16")
    assert_close("S after expiry", np64(S), S_ref, "bf16")


def test_backward_first_wait_expires_then_recovers(cuda_ok):
    B, H, T = 1, 4, 320
    d = workload.make_small(B, H, T, 128, 128, mode="gdn2", dtype="bf16", seed=24, g_scale=0.1, s0_std=0.05)
    gen = torch.Generator().manual_seed(25)
    dO = torch.randn(B, H, T, 128, generator=gen).to(torch.bfloat16)
    dST = torch.randn(B, H, 128, 128, generator=gen)
    dd = to_dev(d)
    run = lambda: gdr.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], dO.cuda(),
                                dST.cuda(), mode="gdn2")
    assert expire_once(run) == TIMEOUT
    out = run()
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(stream()) == 0
    ref = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode="gdn2")
    for n in ("dq", "dk", "dv", "dg", "db", "dw", "dS0"):
        assert_close(f"{n} after expiry", np64(out[n]), ref[n], "bf16")


@pytest.mark.parametrize("nseg", [1, 3])
def test_two_phase_first_wait_expires_then_recovers(cuda_ok, nseg):
    # the state pass's first wait (for its first chunk record) gives up after one poll
    d_cpu = workload.make_small(2, 3, 640, 128, 128, mode="gdn2", dtype="bf16", seed=26, g_scale=0.1,
                                s0_std=0.05)
    d = to_dev(d_cpu)
    run = lambda: gdr.chunk_fwd_two_phase(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                          mode="gdn2", nseg=nseg)
    assert expire_once(run) == TIMEOUT
    o, ST = run()
    torch.cuda.synchronize()
    assert gdr.gdr_last_device_error(stream()) == 0
    o_ref, S_ref = oracle.fwd(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["g"], d_cpu["b"], d_cpu["w"],
                              d_cpu["S0"], mode="gdn2")
    assert_close("o after expiry", np64(o), o_ref, "bf16")
    assert_close("S_T after expiry", np64(ST), S_ref, "bf16")
