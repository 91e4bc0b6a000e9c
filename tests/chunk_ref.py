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


def chunk_records(q, k, v, g, b, w, mode, C=64):
    """Phase one of the two-phase forward: for every chunk of every sequence-head, the factors
    that do not depend on the state, in the pages' W/U form with the decay folded in
    (Kh = b.k.e^gamma, Qg = q.e^gamma, Kb = k.e^-gamma):

      T = (I + strictly_lower(Kh Kb^T))^-1,  W = T Kh,  U = T (w.v),  P = tril(Qg Kb^T)

    Returns records[b][h] = list over chunks of (W, U, Qg, Kb, P, e^gamma_C)."""
    q, k, v, g, b, w = map(_f64, (q, k, v, g, b, w))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    g, b, w = expand_gates(g, b, w, mode, dk, dv)
    recs = [[[] for _ in range(H)] for _ in range(B)]
    for bi in range(B):
        for hi in range(H):
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                n = min(T, c0 + C) - c0
                e = np.exp(np.cumsum(g[bi, hi, sl], axis=0))
                Kh = b[bi, hi, sl] * k[bi, hi, sl] * e
                Qg = q[bi, hi, sl] * e
                Kb = k[bi, hi, sl] / e
                A = np.tril(Kh @ Kb.T, -1)
                Tm = solve_triangular(np.eye(n) + A, np.eye(n), lower=True, unit_diagonal=True)
                recs[bi][hi].append((Tm @ Kh, Tm @ (w[bi, hi, sl] * v[bi, hi, sl]), Qg, Kb,
                                     np.tril(Qg @ Kb.T), e[-1]))
    return recs


def state_pass(recs, S, with_u=True, out=None):
    """Phase two over a run of chunk records from state S: E = U - W S (-W S for a
    transition-map run, which has no write term), O = Qg S + P E, S' = diag(e^gamma_C)
    (S + Kb^T E).  Writes each chunk's O into the list `out` when given; returns S."""
    for W, U, Qg, Kb, P, egc in recs:
        E = (U if with_u else 0.0) - W @ S
        if out is not None:
            out.append(Qg @ S + P @ E)
        S = egc[:, None] * (S + Kb.T @ E)
    return S


def chunk_fwd_two_phase(q, k, v, g, b, w=None, S0=None, mode="gdn2", C=64, nseg=1):
    """The two-phase forward as the library composes it: the records of every chunk first;
    then, with nseg > 1, a sequence split of the state pass over whole-chunk segments
    (seg_chunks = ceil(nchunks / nseg) chunks each): the end state of every segment but the
    last from its own start (S0 for the first, zero for the others), the transition map M_s
    of every inner segment (the state pass from the identity with no write term), the chain
    S_start(s+1) = M_s S_start(s) + S_local(s), and the output pass of every segment from its
    chained start state."""
    B, H, T = q.shape[0], q.shape[1], q.shape[2]
    dk, dv = q.shape[3], v.shape[3]
    recs = chunk_records(q, k, v, g, b, w, mode, C)
    S0 = _f64(S0)
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    nch = (T + C - 1) // C
    nseg = max(1, min(nseg, nch))
    sc = (nch + nseg - 1) // nseg
    nseg = (nch + sc - 1) // sc
    for bi in range(B):
        for hi in range(H):
            r = recs[bi][hi]
            segs = [r[s * sc:(s + 1) * sc] for s in range(nseg)]
            start = np.zeros((dk, dv)) if S0 is None else S0[bi, hi].copy()
            starts = [start]
            for s in range(nseg - 1):
                local = state_pass(segs[s], start if s == 0 else np.zeros((dk, dv)))
                if s == 0:
                    starts.append(local)
                else:
                    M = state_pass(segs[s], np.eye(dk), with_u=False)
                    starts.append(M @ starts[-1] + local)
            out = []
            for s in range(nseg):
                S = state_pass(segs[s], starts[s], out=out)
            o[bi, hi] = np.vstack(out)
            ST[bi, hi] = S
    return o, ST
