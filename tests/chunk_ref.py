"""numpy fp64 chunkwise rederivation of the gated delta rule forward.

An independent second derivation used to pin the sequential oracle: the pages
state that absorbing the cumulative channel-wise decay into the rank-one erase
factor turns the recurrence into a decay-normalised delta recurrence whose
chunkwise WY form is an exact reorganisation (Gated DeltaNet-2 Q&A page, Q4;
Gated DeltaNet-2 Review §3-2.5, "Chunkwise WY training").  This module writes
that form out with plain numpy on one chunk at a time:

  gamma_r = sum_{i<=r} g_i                      (chunk-local, per d_k channel)
  A_ij    = sum_c b_ic k_ic k_jc exp(gamma_ic - gamma_jc),   j < i
  P_ij    = sum_c q_ic k_jc exp(gamma_ic - gamma_jc),        j <= i
  Tm      = (I + A)^-1                          (triangular solve)
  W       = Tm (b . k . exp(gamma)),   U = Tm (w . v)
  E       = U - W S_c                           (the per-token delta errors)
  O       = (q . exp(gamma)) S_c + P E
  S_{c+1} = diag(exp(gamma_C)) S_c + (k . exp(gamma_C - gamma))^T E

Nothing here is shared with the oracle (a per-token loop in C) or with the
CUDA library.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def expand_gates(g, b, w, mode, dk, dv):
    """Full per-channel gates from a mode's tied parameters."""
    if mode == "gdn2":
        return g, b, w
    if mode == "bonly":    # channel erase, one write scalar per token
        return g, b, np.repeat(w[..., None], dv, axis=-1)
    if mode == "wonly":    # one erase scalar per token, channel write
        return g, np.repeat(b[..., None], dk, axis=-1), w
    beta = b
    bb = np.repeat(beta[..., None], dk, axis=-1)
    ww = np.repeat(beta[..., None], dv, axis=-1)
    gg = np.repeat(g[..., None], dk, axis=-1) if mode == "gdn" else g
    return gg, bb, ww


def chunk_fwd(q, k, v, g, b, w=None, S0=None, mode="gdn2", C=64):
    q, k, v, g, b, w, S0 = map(_f64, (q, k, v, g, b, w, S0))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    g, b, w = expand_gates(g, b, w, mode, dk, dv)
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for hi in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, hi].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                qc, kc, vc = q[bi, hi, sl], k[bi, hi, sl], v[bi, hi, sl]
                gc, bc, wc = g[bi, hi, sl], b[bi, hi, sl], w[bi, hi, sl]
                n = qc.shape[0]
                gam = np.cumsum(gc, axis=0)
                ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
                diff = gam[:, None, :] - gam[None, :, :]
                low = (ii >= jj)[..., None]
                dec = np.where(low, np.exp(np.where(low, diff, 0.0)), 0.0)
                A = np.einsum("ic,jc,ijc->ij", bc * kc, kc, dec) * (ii > jj)
                P = np.einsum("ic,jc,ijc->ij", qc, kc, dec) * (ii >= jj)
                eye = np.eye(n)
                Tm = solve_triangular(eye + A, eye, lower=True, unit_diagonal=True)
                W = Tm @ (bc * kc * np.exp(gam))
                U = Tm @ (wc * vc)
                E = U - W @ S
                o[bi, hi, sl] = (qc * np.exp(gam)) @ S + P @ E
                S = np.exp(gam[-1])[:, None] * S + (kc * np.exp(gam[-1][None, :] - gam)).T @ E
            ST[bi, hi] = S
    return o, ST


def chunk_fwd_factorised(q, k, v, g, b, w=None, S0=None, mode="gdn2", C=64):
    """The same forward in the factorised form the tensor-core kernel runs on chunks whose
    cumulative decay stays within e^+-60: no per-pair decays, the decay folded into three
    operands instead (Kh = b.k.e^gamma, Qg = q.e^gamma, Kb = k.e^-gamma) and the state scaled
    after its update:

      [A; P] = [Kh; Qg] Kb^T  (A strictly lower, P lower incl.)    T = (I + A)^-1
      E = T (w.v - Kh S)      O = Qg S + P E      S' = diag(e^gamma_C) (S + Kb^T E)
    """
    q, k, v, g, b, w, S0 = map(_f64, (q, k, v, g, b, w, S0))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    g, b, w = expand_gates(g, b, w, mode, dk, dv)
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for hi in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, hi].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                n = min(T, c0 + C) - c0
                e = np.exp(np.cumsum(g[bi, hi, sl], axis=0))
                Kh = b[bi, hi, sl] * k[bi, hi, sl] * e
                Qg = q[bi, hi, sl] * e
                Kb = k[bi, hi, sl] / e
                AP = np.vstack([Kh, Qg]) @ Kb.T
                A, P = np.tril(AP[:n], -1), np.tril(AP[n:])
                Tm = solve_triangular(np.eye(n) + A, np.eye(n), lower=True, unit_diagonal=True)
                E = Tm @ (w[bi, hi, sl] * v[bi, hi, sl] - Kh @ S)
                o[bi, hi, sl] = Qg @ S + P @ E
                S = e[-1][:, None] * (S + Kb.T @ E)
            ST[bi, hi] = S
    return o, ST
