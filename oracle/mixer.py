"""fp64 oracle of the token mixer's prologue and epilogue around the recurrence --
TEST INFRASTRUCTURE (imported only by tests/ and the benchmark's CPU-baseline leg).

Gated DeltaNet-2 Review §4-3 ("Engineering notes") describes the block around the
recurrence: the q and k paths end in L2 normalisation, the decay branch is a log-decay
projection kept in fp32, the erase and write gates are separate projections through a
sigmoid, and the recurrent output is RMS-normalised and multiplied by a SiLU output gate
before the output projection.  The readings taken where the page is silent:

  q_hat = q / sqrt(sum_d q_d^2 + 1e-6)               (same for k; per token and head)
  g     = -softplus(x_g)                             (natural-log decay, <= 0)
  b     = b_range * sigmoid(x_b),  w = sigmoid(x_w)   (b_range 2: expanded erase range)
  y     = o / sqrt(mean_v o_v^2 + eps) * weight * z * sigmoid(z)
                                                     (weight [dv] shared by the heads)

Inputs may be laid out head-major [B, H, T, .] or token-major [B, T, H, .]; the
recurrence itself is the oracle of gdr_oracle.c (oracle.fwd).  Plain torch float64 CPU
operations, one definition per line.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

L2_EPS = 1e-6


def _t64(x):
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        return torch.from_numpy(x).double()
    return x.detach().cpu().double()


def l2norm(x):
    """x / sqrt(sum over the last axis of x^2 + 1e-6)."""
    return x / torch.sqrt((x * x).sum(-1, keepdim=True) + L2_EPS)


def softplus(x):
    """log(1 + exp(x)), computed as max(x, 0) + log1p(exp(-|x|))."""
    return torch.clamp(x, min=0) + torch.log1p(torch.exp(-torch.abs(x)))


def sigmoid(x):
    return 1.0 / (1.0 + torch.exp(-x))


def rmsnorm_gate(o, z, weight, eps):
    """o / sqrt(mean over the last axis of o^2 + eps) * weight * z * sigmoid(z)."""
    rstd = 1.0 / torch.sqrt((o * o).mean(-1, keepdim=True) + eps)
    return o * rstd * weight * (z * sigmoid(z))


def prologue(q, k, v, xg, xb, xw, b_range=1.0):
    """Activated recurrence inputs (head-major, float64 tensors)."""
    q, k, v, xg, xb, xw = map(_t64, (q, k, v, xg, xb, xw))
    return dict(q=l2norm(q), k=l2norm(k), v=v, g=-softplus(xg), b=b_range * sigmoid(xb),
                w=None if xw is None else sigmoid(xw))


def to_head_major(x):
    """[B, T, H, ...] -> [B, H, T, ...]"""
    return None if x is None else x.transpose(1, 2).contiguous()


def mixer_fwd(q, k, v, xg, xb, xw, z, weight, S0=None, mode="gdn2", eps=1e-5, b_range=1.0,
              token_major=False):
    """Prologue, recurrence (oracle.fwd) and epilogue.  Returns (y, S_T) as float64 numpy
    arrays, y in the layout of the inputs."""
    args = [_t64(a) for a in (q, k, v, xg, xb, xw, z)]
    if token_major:
        args = [to_head_major(a) for a in args]
    q, k, v, xg, xb, xw, z = args
    a = prologue(q, k, v, xg, xb, xw, b_range)
    o, ST = oracle.fwd(a["q"], a["k"], a["v"], a["g"], a["b"], a["w"], S0, mode=mode)
    y = rmsnorm_gate(torch.from_numpy(o), z, _t64(weight), eps)
    if token_major:
        y = y.transpose(1, 2).contiguous()
    return y.numpy(), ST
