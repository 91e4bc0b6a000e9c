"""Seeded synthetic inputs for the gated delta rule forward.

This module only draws random tensors and prepares them the way the token-mixer
block of the pages prepares its inputs (q/k L2-normalised per token, log-decay
as -softplus, erase/write gates as sigmoid; Gated DeltaNet-2 Review §4-3 and
Gated DeltaNet review §3-2.2).  It holds none of the recurrence's arithmetic,
so both the CUDA path and the oracle may consume what it produces.

Layouts (row-major, contiguous):
  q, k          [B, H, T, dk]
  v             [B, H, T, dv]
  g_log         [B, H, T, dk] fp32   (GDN mode: [B, H, T])
  b             [B, H, T, dk]        (KDA / GDN modes: beta, [B, H, T]; w-only: [B, H, T])
  w             [B, H, T, dv]        (KDA / GDN modes: None; b-only: [B, H, T])
  S0            [B, H, dk, dv] fp32 or None
q, k, v, b, w are rounded to the workload's dtype (fp32 or bf16); g_log and S0
are always fp32.  Draw order from one torch CPU generator: q, k, v, g, b (or
beta), w, S0, then any extra tied-mode beta or variant scalar gate.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

MODES = ("gdn2", "kda", "gdn", "bonly", "wonly")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str            # "f32" or "bf16": dtype of q, k, v, b, w, o
    mode: str             # "gdn2", "kda" or "gdn" (the variants derive from "gdn2")
    seed: int
    g_scale: float = 0.1  # g_log = -softplus(N(0,1)) * g_scale
    q_scale: bool = False # multiply q by dk**-0.5 after normalisation
    s0_std: float = 0.0   # 0 => S0 = None (zeros)
    extra: dict = field(default_factory=dict)

    @property
    def units(self) -> int:
        """Token-heads processed by one forward call."""
        return self.B * self.H * self.T


# The five workloads the method is measured on.  Shapes follow the training
# recipe of the pages (16 heads, d_k = d_v = 128, sequence 2K-16K; Gated
# DeltaNet-2 Review §4-2) with synthetic data standing in for FineWeb-Edu.
CONFIGS = {
    "gdn2_tiny": Workload("gdn2_tiny", B=1, H=1, T=256, dk=64, dv=64, chunk=64,
                          dtype="f32", mode="gdn2", seed=0, g_scale=1.0,
                          q_scale=True, s0_std=0.0),
    "gdn_t2k": Workload("gdn_t2k", B=4, H=16, T=2048, dk=128, dv=128, chunk=64,
                        dtype="bf16", mode="gdn", seed=1, g_scale=0.1, s0_std=0.0),
    "gdn2_t4k": Workload("gdn2_t4k", B=8, H=16, T=4096, dk=128, dv=128, chunk=64,
                         dtype="bf16", mode="gdn2", seed=2, g_scale=0.1, s0_std=0.02),
    "gdn2_t16k": Workload("gdn2_t16k", B=1, H=16, T=16384, dk=128, dv=128, chunk=64,
                          dtype="bf16", mode="gdn2", seed=3, g_scale=0.1, s0_std=0.02),
}

# Batched decode: 256 sequences x 16 heads, one token per step, a pool of 64
# distinct seeded steps cycled over 1000 steps.
DECODE = dict(name="gdn2_decode", N=256, H=16, dk=128, dv=128, dtype="bf16",
              mode="gdn2", seed=4, g_scale=0.1, s0_std=0.02, steps=1000, pool=64)


def torch_dtype(dtype: str) -> torch.dtype:
    if dtype == "f32":
        return torch.float32
    if dtype == "bf16":
        return torch.bfloat16
    raise ValueError(f"unknown dtype {dtype!r}")


def _l2norm(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    return x * torch.rsqrt((x * x).sum(-1, keepdim=True) + eps)


def make_inputs(wl: Workload, mode: Optional[str] = None, B: Optional[int] = None,
                b_range: float = 1.0):
    """Draw one workload's inputs on the CPU.  Returns a dict of torch tensors.

    `mode` overrides the workload's mode (the tied KDA variant of the long
    context workload uses the same q, k, v, g and draws beta after S0; the b-only
    and w-only gate-ablation variants of a GDN-2 workload draw their scalar gate
    there too).  `b_range` scales the erase gate: 2 gives the expanded erase range
    b in [0, 2] of the same ablation.
    `B` draws only the first B sequences' worth of shapes (used by sharded
    runs; the draw is then a different sample)."""
    mode = mode or wl.mode
    assert mode in MODES
    Bn = wl.B if B is None else B
    gen = torch.Generator().manual_seed(wl.seed)
    H, T, dk, dv = wl.H, wl.T, wl.dk, wl.dv
    dt = torch_dtype(wl.dtype)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _l2norm(randn(Bn, H, T, dk))
    if wl.q_scale:
        q = q * (dk ** -0.5)
    k = _l2norm(randn(Bn, H, T, dk))
    v = randn(Bn, H, T, dv)
    if wl.mode == "gdn":
        g = -torch.nn.functional.softplus(randn(Bn, H, T)) * wl.g_scale
    else:
        g = -torch.nn.functional.softplus(randn(Bn, H, T, dk)) * wl.g_scale
    if wl.mode == "gdn2":
        b = torch.sigmoid(randn(Bn, H, T, dk))
        w = torch.sigmoid(randn(Bn, H, T, dv))
    else:
        b = torch.sigmoid(randn(Bn, H, T))   # beta
        w = None
    S0 = randn(Bn, H, dk, dv) * wl.s0_std if wl.s0_std > 0 else None
    if mode == "kda" and wl.mode == "gdn2":
        # tied variant on the same q, k, v, g: b = w = beta * 1
        b = torch.sigmoid(randn(Bn, H, T))
        w = None
    elif mode == "bonly":
        w = torch.sigmoid(randn(Bn, H, T))   # scalar write gate
    elif mode == "wonly":
        b = torch.sigmoid(randn(Bn, H, T))   # scalar erase gate
    b = b * b_range
    out = dict(q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
               g=g.contiguous(), b=b.to(dt).contiguous(),
               w=None if w is None else w.to(dt).contiguous(),
               S0=None if S0 is None else S0.contiguous(), mode=mode)
    return out


def make_small(B, H, T, dk, dv, mode="gdn2", dtype="f32", seed=0, g_scale=1.0,
               s0_std=0.0, g_const=None, b_range=1.0):
    """Inputs for a small parity case of arbitrary shape."""
    wl = Workload("small", B=B, H=H, T=T, dk=dk, dv=dv, chunk=64, dtype=dtype,
                  mode="gdn" if mode == "gdn" else "gdn2", seed=seed,
                  g_scale=g_scale, s0_std=s0_std)
    d = make_inputs(wl, mode=mode, b_range=b_range)
    if g_const is not None:
        d["g"] = torch.full_like(d["g"], float(g_const))
    return d


def make_decode_pool(cfg=DECODE, N=None, pool=None):
    """Decode workload: a pool of `pool` distinct steps plus the initial state.

    Returns dict(q, k, v, g, b, w) each [pool, N, H, d] and S0 [N, H, dk, dv]."""
    N = cfg["N"] if N is None else N
    P = cfg["pool"] if pool is None else pool
    H, dk, dv = cfg["H"], cfg["dk"], cfg["dv"]
    gen = torch.Generator().manual_seed(cfg["seed"])
    dt = torch_dtype(cfg["dtype"])

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _l2norm(randn(P, N, H, dk))
    k = _l2norm(randn(P, N, H, dk))
    v = randn(P, N, H, dv)
    g = -torch.nn.functional.softplus(randn(P, N, H, dk)) * cfg["g_scale"]
    b = torch.sigmoid(randn(P, N, H, dk))
    w = torch.sigmoid(randn(P, N, H, dv))
    S0 = randn(N, H, dk, dv) * cfg["s0_std"]
    return dict(q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
                g=g.contiguous(), b=b.to(dt).contiguous(), w=w.to(dt).contiguous(),
                S0=S0.contiguous(), mode=cfg["mode"])


# The token-mixer workload: the raw projections of the T=4K shape, token-major as a
# block's projections produce them.  xg ~ N(-2.5, 1) puts the decay g = -softplus(xg)
# near the T=4K workload's typical size (about -0.1 per token).
MIXER = dict(name="mixer_t4k", B=8, H=16, T=4096, dk=128, dv=128, chunk=64, mode="gdn2",
             layout="bthd", seed=5, xg_shift=-2.5, s0_std=0.02)


def make_mixer_inputs(B, H, T, dk, dv, mode="gdn2", layout="bhtd", seed=0, xg_shift=-2.5,
                      xg_scale=1.0, s0_std=0.0, b_range=1.0):
    """Raw inputs of the token-mixer block (gdr_mixer_fwd): q, k, v, the pre-activation
    gates xg (fp32), xb, xw, the output gate z (bf16) and the RMSNorm weight (fp32 [dv]).
    layout "bhtd" draws [B, H, T, .], "bthd" draws [B, T, H, .].  Draw order from one
    torch CPU generator: q, k, v, xg, xb, xw, S0, z, weight."""
    assert mode in MODES and layout in ("bhtd", "bthd")
    gen = torch.Generator().manual_seed(seed)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    lead = (B, H, T) if layout == "bhtd" else (B, T, H)
    q = randn(*lead, dk)
    k = randn(*lead, dk)
    v = randn(*lead, dv)
    xg = (randn(*lead) if mode == "gdn" else randn(*lead, dk)) * xg_scale + xg_shift
    xb = randn(*lead, dk) if mode in ("gdn2", "bonly") else randn(*lead)
    if mode in ("gdn2", "wonly"):
        xw = randn(*lead, dv)
    elif mode == "bonly":
        xw = randn(*lead)
    else:
        xw = None
    S0 = randn(B, H, dk, dv) * s0_std if s0_std > 0 else None
    z = randn(*lead, dv)
    weight = 1.0 + 0.1 * randn(dv)
    bf = lambda x: None if x is None else x.to(torch.bfloat16).contiguous()
    return dict(q=bf(q), k=bf(k), v=bf(v), xg=xg.contiguous(), xb=bf(xb), xw=bf(xw), z=bf(z),
                weight=weight.contiguous(), S0=None if S0 is None else S0.contiguous(), mode=mode,
                layout=layout, b_range=b_range)


def shard_range(n_units: int, rank: int, world: int):
    """Contiguous [lo, hi) share of n_units for one rank (independent units)."""
    base, rem = divmod(n_units, world)
    lo = rank * base + min(rank, rem)
    hi = lo + base + (1 if rank < rem else 0)
    return lo, hi
