"""GPU parity of gdr_decode_step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workload
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu


def pool_step(pool, p, sel=None):
    out = {}
    for k in ("q", "k", "v", "g", "b", "w"):
        x = pool[k][p]
        out[k] = x if sel is None else x[sel]
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (16, 128), (32, 16)])
def test_decode_small(cuda_ok, dtype, mode, dk, dv):
    torch.manual_seed(dk * dv)
    N, H = 5, 3
    d = workload.make_small(N, H, 1, dk, dv, mode=mode, dtype=dtype, seed=dk + dv, s0_std=0.2)
    S0 = torch.randn(N, H, dk, dv) * 0.2
    sq = lambda x: None if x is None else x[:, :, 0].contiguous()
    args = [sq(d[k]) for k in ("q", "k", "v", "g", "b", "w")]
    o_ref, S_ref = oracle.decode(*args, S=S0, mode=mode)
    dev = [None if a is None else a.cuda() for a in args]
    S = S0.cuda()
    o = gdr.decode_step(*dev, S, mode=mode)
    torch.cuda.synchronize()
    assert_close("o", np64(o), o_ref, dtype)
    assert_close("S", np64(S), S_ref, "f32" if dtype == "f32" else dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
def test_decode_many_heads(cuda_ok, dtype, mode):
    """More heads than SMs at d = 128: every CTA of the streaming kernel cycles its state
    buffers several times (1177 heads, not a multiple of the SM count), two steps in a row."""
    N, H, d = 107, 11, 128
    dd = workload.make_small(N, H, 2, d, d, mode=mode, dtype=dtype, seed=77, s0_std=0.2)
    S0 = torch.randn(N, H, d, d, generator=torch.Generator().manual_seed(78)) * 0.2
    step = lambda t: [None if dd[k] is None else dd[k][:, :, t].contiguous() for k in ("q", "k", "v", "g", "b", "w")]
    S = S0.cuda()
    Sr = S0.double().numpy()
    for t in range(2):
        args = step(t)
        o = gdr.decode_step(*[None if a is None else a.cuda() for a in args], S, mode=mode)
        o_ref, Sr = oracle.decode(*args, S=Sr, mode=mode)
        torch.cuda.synchronize()
        assert_close(f"o step {t}", np64(o), o_ref, dtype)
    assert_close("S", np64(S), Sr, "f32" if dtype == "f32" else dtype)


def test_decode_workload_1000_steps(cuda_ok):
    cfg = workload.DECODE
    pool = workload.make_decode_pool(cfg)
    P, steps = cfg["pool"], cfg["steps"]
    dpool = to_dev(pool)
    S = dpool["S0"].clone()
    outs = []
    for s in range(steps):
        st = pool_step(dpool, s % P)
        o = gdr.decode_step(st["q"], st["k"], st["v"], st["g"], st["b"], st["w"], S, mode="gdn2")
        if s < P:
            outs.append(o.clone())
    torch.cuda.synchronize()
    assert torch.isfinite(S).all()
    # sampled (sequence, head) pairs; each is independent of the others
    rng = np.random.default_rng(5)
    N, H = cfg["N"], cfg["H"]
    flat = rng.choice(N * H, size=256, replace=False)
    ns, hs = flat // H, flat % H
    Sr = pool["S0"][ns, hs][:, None].double().numpy()
    for s in range(steps):
        st = pool_step(pool, s % P)
        sel = lambda x: x[ns, hs][:, None]
        o_ref, Sr = oracle.decode(sel(st["q"]), sel(st["k"]), sel(st["v"]), sel(st["g"]),
                                  sel(st["b"]), sel(st["w"]), S=Sr, mode="gdn2")
        if s < P:
            assert_close(f"o step {s}", np64(outs[s][ns, hs]), o_ref[:, 0], "bf16", head_axes=1)
    assert_close("S after 1000 steps", np64(S[ns, hs]), Sr[:, 0], "bf16", head_axes=1)
    # the fp32 state itself is carried in fp32 on both sides: check it tightly too
    assert np.max(np.abs(np64(S[ns, hs]) - Sr[:, 0])) < 1e-4
