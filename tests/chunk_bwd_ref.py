"""numpy fp64 transcription of the factorised chunk backward that the tensor-core kernel runs.

The per-chunk gradient kernel of the backward does not form per-pair decays: it works with
the decay folded into three operands, Kh = b.k.e^gamma, Qg = q.e^gamma, Kb = k.e^-gamma, and
a handful of dense products (the chunkwise WY form of Gated DeltaNet-2 Review §3-2.5,
differentiated for the gate-aware backward of §4-3).  Per 64-token chunk, with S the state
at its start and dS' the gradient of the state at its end, dS~ = diag(e^gamma_C) dS':

  A = strict_lower(Kh Kb^T)     P = lower_incl(Qg Kb^T)     T = (I + A)^-1
  E = T (w.v - Kh S)
  dE = Kb dS~ + P^T dO          dR = T^T dE
  dA = strict_lower(-dR E^T)    (= strict_lower(-T^T (dE R^T) T^T), with R = T^-1 E)
  dP = strict_lower(dO E^T),    its diagonal d_t = <dO_t, E_t> kept apart
  dKh = -dR S^T + dA Kb         dQg = dO S^T + dP Kb
  dKb = dA^T Kh + dP^T Qg       dKe = E dS~^T
  dq = dQg e^gamma + d k        dk = dKh b e^gamma + (dKb + dKe) e^-gamma + d q
  db = dKh k e^gamma            dgamma = dQg Qg + dKh Kh - (dKb + dKe) Kb
  dgamma_C = sum_v S dS~ + sum_t dKe Kb
  dg = dgamma_C + reverse cumulative sum of dgamma;   dv = dR w,  dw = dR v

The states at the chunk starts and the state gradients at the chunk ends come from plain
per-chunk passes written here as well.  Used by the CPU tests to pin this algebra against
the adjoint oracle; nothing is shared with the oracle or the CUDA library.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

import chunk_ref


def _pad(x, Tp):
    if x is None:
        return None
    out = np.zeros((Tp,) + x.shape[1:], dtype=np.float64)
    out[: x.shape[0]] = x
    return out


def chunk_bwd_head(q, k, v, g, b, w, S0, dO, dST, C=64, keep_diagonal=True):
    """One sequence-head with full per-channel gates: q, k, b, g [T, dk]; v, w, dO [T, dv];
    S0, dST [dk, dv].  Returns dq, dk, dv, dg, db, dw (per channel) and dS0.
    keep_diagonal=False drops dP's diagonal terms (a planted mistake for the tests)."""
    T, dk = q.shape
    dv = v.shape[1]
    nc = (T + C - 1) // C
    Tp = nc * C
    q, k, b, g, v, w, dO = (_pad(x, Tp) for x in (q, k, b, g, v, w, dO))
    gam = np.zeros_like(g)
    ops = []
    for c in range(nc):
        sl = slice(c * C, (c + 1) * C)
        gm = np.cumsum(g[sl], axis=0)
        e = np.exp(gm)
        Kh, Qg, Kb = b[sl] * k[sl] * e, q[sl] * e, k[sl] / e
        A = np.tril(Kh @ Kb.T, -1)
        P = np.tril(Qg @ Kb.T)
        Tm = solve_triangular(np.eye(C) + A, np.eye(C), lower=True, unit_diagonal=True)
        gam[sl] = gm
        ops.append((Kh, Qg, Kb, P, Tm, gm[-1]))
    # states at the chunk starts (forward) and state gradients at the chunk ends (reverse)
    S = [S0.copy()]
    for c in range(nc):
        Kh, Qg, Kb, P, Tm, gC = ops[c]
        sl = slice(c * C, (c + 1) * C)
        E = Tm @ (w[sl] * v[sl] - Kh @ S[c])
        S.append(np.exp(gC)[:, None] * S[c] + (Kb * np.exp(gC)).T @ E)
    dS = [None] * (nc + 1)
    dS[nc] = dST.copy()
    for c in range(nc - 1, -1, -1):
        Kh, Qg, Kb, P, Tm, gC = ops[c]
        sl = slice(c * C, (c + 1) * C)
        dE = (Kb * np.exp(gC)) @ dS[c + 1] + P.T @ dO[sl]
        dR = Tm.T @ dE
        dS[c] = np.exp(gC)[:, None] * dS[c + 1] + Qg.T @ dO[sl] - Kh.T @ dR
    # per-chunk gradients in the factorised form
    out = {n: np.zeros((Tp, dk)) for n in ("dq", "dk", "db", "dg")}
    out.update({n: np.zeros((Tp, dv)) for n in ("dv", "dw")})
    for c in range(nc):
        Kh, Qg, Kb, P, Tm, gC = ops[c]
        sl = slice(c * C, (c + 1) * C)
        Sc, egc = S[c], np.exp(gC)
        dSt = egc[:, None] * dS[c + 1]
        E = Tm @ (w[sl] * v[sl] - Kh @ Sc)
        dE = Kb @ dSt + P.T @ dO[sl]
        dR = Tm.T @ dE
        G = np.vstack([-dR, dO[sl]]) @ E.T
        dA = np.tril(G[:C], -1)
        dP_full = G[C:]
        dPd = np.diag(dP_full).copy() if keep_diagonal else np.zeros(C)
        dP = np.tril(dP_full, -1)
        dKh = -dR @ Sc.T + dA @ Kb
        dQg = dO[sl] @ Sc.T + dP @ Kb
        dKb = dA.T @ Kh + dP.T @ Qg
        dKe = E @ dSt.T
        e = np.exp(gam[sl])
        out["dq"][sl] = dQg * e + dPd[:, None] * k[sl]
        out["dk"][sl] = dKh * b[sl] * e + (dKb + dKe) / e + dPd[:, None] * q[sl]
        out["db"][sl] = dKh * k[sl] * e
        dgam = dQg * Qg + dKh * Kh - (dKb + dKe) * Kb
        dgC = np.sum(Sc * dSt, axis=1) + np.sum(dKe * Kb, axis=0)
        out["dg"][sl] = dgC[None, :] + np.cumsum(dgam[::-1], axis=0)[::-1]
        out["dv"][sl] = dR * w[sl]
        out["dw"][sl] = dR * v[sl]
    res = {n: x[:T] for n, x in out.items()}
    res["dS0"] = dS[0]
    return res


def chunk_bwd(q, k, v, g, b, w=None, S0=None, dO=None, dST=None, mode="gdn2", C=64, keep_diagonal=True):
    """[B, H, T, .] inputs as the library takes them; returns the gradients in the same
    shapes as the oracle's backward (scalar gates summed over the channels they stand for)."""
    f = chunk_ref._f64
    q, k, v, g, b, w, S0, dO, dST = (f(x) for x in (q, k, v, g, b, w, S0, dO, dST))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out = {n: [] for n in ("dq", "dk", "dv", "dg", "db", "dw", "dS0")}
    for bi in range(B):
        for h in range(H):
            gg, bb, ww = chunk_ref.expand_gates(g[bi, h], b[bi, h], None if w is None else w[bi, h], mode, dk, dv)
            r = chunk_bwd_head(q[bi, h], k[bi, h], v[bi, h], gg, bb, ww,
                               np.zeros((dk, dv)) if S0 is None else S0[bi, h], dO[bi, h],
                               np.zeros((dk, dv)) if dST is None else dST[bi, h], C=C,
                               keep_diagonal=keep_diagonal)
            db, dw, dgv = r["db"], r["dw"], r["dg"]
            if mode in ("kda", "gdn"):      # beta is both gates
                db = db.sum(-1) + dw.sum(-1)
                dw = None
            elif mode == "wonly":           # scalar erase gate
                db = db.sum(-1)
            elif mode == "bonly":           # scalar write gate
                dw = dw.sum(-1)
            if mode == "gdn":
                dgv = dgv.sum(-1)
            for n, x in (("dq", r["dq"]), ("dk", r["dk"]), ("dv", r["dv"]), ("dg", dgv), ("db", db),
                         ("dw", dw), ("dS0", r["dS0"])):
                out[n].append(x)
    shp = lambda lst: None if lst[0] is None else np.stack(lst).reshape((B, H) + lst[0].shape)
    return {n: shp(lst) for n, lst in out.items()}
