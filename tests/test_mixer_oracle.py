"""Pins for the mixer oracle (oracle/mixer.py): each activation against a closed form or
an identity, the epilogue against its definition on special rows, the layouts against
each other, and the wiring against the recurrence oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workload
from oracle import mixer


def test_l2norm_closed_form():
    x = torch.randn(5, 7, 33, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    y = mixer.l2norm(x)
    n = torch.sqrt((x * x).sum(-1))
    np.testing.assert_allclose(torch.sqrt((y * y).sum(-1)), n / torch.sqrt(n * n + 1e-6), rtol=1e-14)
    cos = (x * y).sum(-1) / (n * torch.sqrt((y * y).sum(-1)))
    np.testing.assert_allclose(cos, np.ones_like(cos), rtol=1e-14)
    assert torch.all(mixer.l2norm(torch.zeros(3, 8, dtype=torch.float64)) == 0)


def test_softplus_and_sigmoid_identities():
    xs = [-30.0, -5.5, -1.0, -1e-3, 0.0, 0.25, 2.0, 7.0, 40.0]
    x = torch.tensor(xs, dtype=torch.float64)
    sp = mixer.softplus(x)
    for xi, si in zip(xs, sp.tolist()):      # Python's libm, an independent implementation
        ref = xi + math.log1p(math.exp(-xi)) if xi > 0 else math.log1p(math.exp(xi))
        assert abs(si - ref) <= 1e-15 * max(1.0, abs(ref))
    assert abs(mixer.softplus(torch.tensor(0.0, dtype=torch.float64)).item() - math.log(2.0)) < 1e-16
    np.testing.assert_allclose(sp - mixer.softplus(-x), x, rtol=1e-14, atol=1e-14)
    s = mixer.sigmoid(x)
    np.testing.assert_allclose(s + mixer.sigmoid(-x), np.ones(len(xs)), rtol=1e-15)
    assert mixer.sigmoid(torch.tensor(0.0, dtype=torch.float64)).item() == 0.5


def test_rmsnorm_gate_special_rows():
    dv, eps = 16, 1e-5
    w = torch.linspace(0.5, 1.5, dv, dtype=torch.float64)
    c = 0.3
    o = torch.full((2, dv), c, dtype=torch.float64)
    z = torch.full((2, dv), 2.0, dtype=torch.float64)
    y = mixer.rmsnorm_gate(o, z, w, eps)
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    np.testing.assert_allclose(y, (c / math.sqrt(c * c + eps)) * w * silu2 * torch.ones(2, dv), rtol=1e-14)
    # SiLU(0) = 0 closes the gate
    assert torch.all(mixer.rmsnorm_gate(o, torch.zeros_like(z), w, eps) == 0)
    # without eps the normalisation is scale-free
    r = torch.randn(3, dv, generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    np.testing.assert_allclose(mixer.rmsnorm_gate(7.5 * r, z[:1], w, 0.0), mixer.rmsnorm_gate(r, z[:1], w, 0.0),
                               rtol=1e-13)


def _raw(seed, B, H, T, dk, dv, mode):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    sg = (B, H, T) if mode == "gdn" else (B, H, T, dk)
    sb = (B, H, T, dk) if mode in ("gdn2", "bonly") else (B, H, T)
    sw = (B, H, T, dv) if mode in ("gdn2", "wonly") else ((B, H, T) if mode == "bonly" else None)
    return dict(q=r(B, H, T, dk), k=r(B, H, T, dk), v=r(B, H, T, dv), xg=r(*sg) - 2.0, xb=r(*sb),
                xw=None if sw is None else r(*sw), z=r(B, H, T, dv), weight=1.0 + 0.1 * r(dv),
                S0=0.1 * r(B, H, dk, dv))


@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
def test_mixer_wiring_and_layouts(mode):
    B, H, T, dk, dv = 2, 3, 21, 8, 6
    d = _raw(5, B, H, T, dk, dv, mode)
    y, ST = mixer.mixer_fwd(d["q"], d["k"], d["v"], d["xg"], d["xb"], d["xw"], d["z"], d["weight"],
                            d["S0"], mode=mode, eps=1e-5)
    # wiring: activations written out here, recurrence by the sequential oracle
    nrm = lambda x: x / np.sqrt((x ** 2).sum(-1, keepdims=True) + 1e-6)
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    n = lambda x: None if x is None else x.numpy()
    o, ST2 = oracle.fwd(nrm(n(d["q"])), nrm(n(d["k"])), n(d["v"]), -np.log1p(np.exp(n(d["xg"]))),
                        sig(n(d["xb"])), None if d["xw"] is None else sig(n(d["xw"])), n(d["S0"]), mode=mode)
    rstd = 1.0 / np.sqrt((o ** 2).mean(-1, keepdims=True) + 1e-5)
    zz = n(d["z"])
    np.testing.assert_allclose(y, o * rstd * n(d["weight"]) * zz * sig(zz), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ST, ST2, rtol=1e-13, atol=1e-14)
    # token-major inputs give the token-major transpose of the same result
    tm = lambda x: None if x is None else x.transpose(1, 2).contiguous()
    y2, ST3 = mixer.mixer_fwd(*(tm(d[x]) for x in ("q", "k", "v", "xg", "xb", "xw", "z")), d["weight"],
                              d["S0"], mode=mode, eps=1e-5, token_major=True)
    np.testing.assert_allclose(y2, np.swapaxes(y, 1, 2), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(ST3, ST, rtol=1e-14, atol=1e-15)
