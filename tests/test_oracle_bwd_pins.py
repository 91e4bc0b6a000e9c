"""Pins for the backward oracle (oracle.bwd, the adjoint of the sequential recurrence):
central finite differences of the forward oracle in every mode (the loss is
L = sum(o * dO) + sum(S_T * dS_T)), closed forms for causal linear attention and for a pure
decay, and the empty sequence.  None of these reuses the adjoint's own arithmetic."""
import numpy as np
import pytest

import oracle

MODES = ["gdn2", "kda", "gdn", "bonly", "wonly"]


def tiny(mode, B=1, H=2, T=37, dk=3, dv=4, seed=0, s0=True):
    rng = np.random.default_rng(seed)
    sg = (B, H, T) if mode == "gdn" else (B, H, T, dk)
    sb = (B, H, T, dk) if mode in ("gdn2", "bonly") else (B, H, T)
    sw = {"gdn2": (B, H, T, dv), "wonly": (B, H, T, dv), "bonly": (B, H, T)}.get(mode)
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    d = dict(q=rng.standard_normal((B, H, T, dk)) * 0.5, k=rng.standard_normal((B, H, T, dk)) * 0.5,
             v=rng.standard_normal((B, H, T, dv)), g=-np.log1p(np.exp(rng.standard_normal(sg))) * 0.5,
             b=sig(rng.standard_normal(sb)), w=None if sw is None else sig(rng.standard_normal(sw)),
             S0=rng.standard_normal((B, H, dk, dv)) * 0.3 if s0 else None)
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    return d, dO, dST


def loss(d, dO, dST, mode):
    o, ST = oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode, nthreads=1)
    return float((o * dO).sum() + (ST * dST).sum())


@pytest.mark.parametrize("mode", MODES)
def test_finite_differences(mode):
    # T = 37 crosses the adjoint's 32-token checkpoint block
    d, dO, dST = tiny(mode)
    g = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode=mode, nthreads=1)
    h = 1e-5
    names = ["q", "k", "v", "g", "b", "S0"] + (["w"] if d["w"] is not None else [])
    for name in names:
        x = d[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = loss(d, dO, dST, mode)
            x[idx] = keep - h
            lm = loss(d, dO, dST, mode)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        ad = g["dS0" if name == "S0" else "d" + name]
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(ad, fd, rtol=0, atol=2e-7 * scale, err_msg=f"{mode} d{name}")


def test_linear_attention_closed_form():
    # g = 0, b = 0, w = 1: o_t = S0^T q_t + sum_{j<=t} (k_j . q_t) v_j and
    # S_T = S0 + sum_j k_j v_j^T, so every gradient is a plain sum
    rng = np.random.default_rng(3)
    B, H, T, dk, dv = 1, 1, 45, 5, 6
    q, k = rng.standard_normal((B, H, T, dk)), rng.standard_normal((B, H, T, dk))
    v, S0 = rng.standard_normal((B, H, T, dv)), rng.standard_normal((B, H, dk, dv))
    g, b, w = np.zeros((B, H, T, dk)), np.zeros((B, H, T, dk)), np.ones((B, H, T, dv))
    dO, dST = rng.standard_normal((B, H, T, dv)), rng.standard_normal((B, H, dk, dv))
    r = oracle.bwd(q, k, v, g, b, w, S0, dO, dST, mode="gdn2", nthreads=1)
    Q, K, V, D, S, G = q[0, 0], k[0, 0], v[0, 0], dO[0, 0], S0[0, 0], dST[0, 0]
    mask = np.tril(np.ones((T, T)))                          # [t, j]: j <= t
    vd = V @ D.T                                             # [j, t] = v_j . dO_t
    dq = D @ S.T + (mask * vd.T) @ K                         # S0 dO_t + sum_{j<=t} k_j (v_j . dO_t)
    dk = (mask.T * vd) @ Q + V @ G.T                         # sum_{t>=j} q_t (v_j . dO_t) + dST v_j
    dv = (mask.T * (K @ Q.T)) @ D + K @ G                    # sum_{t>=j} (k_j . q_t) dO_t + dST^T k_j
    dS0 = Q.T @ D + G
    np.testing.assert_allclose(r["dq"][0, 0], dq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["dk"][0, 0], dk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["dv"][0, 0], dv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["dS0"][0, 0], dS0, rtol=1e-12, atol=1e-12)


def test_pure_decay_closed_form():
    # b = w = 0: S_t = diag(exp(G_t)) S0 with G_t = sum_{s<=t} g_s, nothing is written
    rng = np.random.default_rng(4)
    B, H, T, dk, dv = 1, 1, 40, 4, 3
    q, k, v = rng.standard_normal((B, H, T, dk)), rng.standard_normal((B, H, T, dk)), rng.standard_normal((B, H, T, dv))
    g = -rng.uniform(0.0, 0.3, (B, H, T, dk))
    b, w = np.zeros((B, H, T, dk)), np.zeros((B, H, T, dv))
    S0 = rng.standard_normal((B, H, dk, dv))
    dO, dST = rng.standard_normal((B, H, T, dv)), rng.standard_normal((B, H, dk, dv))
    r = oracle.bwd(q, k, v, g, b, w, S0, dO, dST, mode="gdn2", nthreads=1)
    Q, Dd, S, G = q[0, 0], dO[0, 0], S0[0, 0], dST[0, 0]
    cum = np.exp(np.cumsum(g[0, 0], axis=0))                 # [t, i] = exp(G_t[i])
    St = cum[:, :, None] * S[None]                           # S_t
    np.testing.assert_allclose(r["dq"][0, 0], np.einsum("tij,tj->ti", St, Dd), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["dk"][0, 0], 0.0, atol=1e-13)
    np.testing.assert_allclose(r["dv"][0, 0], 0.0, atol=1e-13)
    # L = sum_t q_t^T S_t dO_t + <S_T, dST>;  dL/dG_t[i] = (q_t[i] (S_t dO_t)[i]) + [t = T-1] (S_T . dST)[i]
    per = Q * np.einsum("tij,tj->ti", St, Dd)
    per[-1] += (St[-1] * G).sum(1)
    dg = np.cumsum(per[::-1], axis=0)[::-1]                  # dL/dg_s = sum_{t>=s} dL/dG_t
    np.testing.assert_allclose(r["dg"][0, 0], dg, rtol=1e-11, atol=1e-12)
    dS0 = np.einsum("ti,tj,ti->ij", cum, Dd, Q) + cum[-1][:, None] * G
    np.testing.assert_allclose(r["dS0"][0, 0], dS0, rtol=1e-12, atol=1e-12)


def test_empty_sequence_and_no_initial_state():
    d, dO, dST = tiny("gdn2", T=0)
    r = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode="gdn2")
    np.testing.assert_array_equal(r["dS0"], dST)
    # without S0 the gradient with respect to the (zero) initial state is still returned
    d, dO, dST = tiny("kda", T=9, s0=False)
    r = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], None, dO, dST, mode="kda")
    d["S0"] = np.zeros((1, 2, 3, 4))
    r2 = oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode="kda")
    for key in ("dq", "dk", "dv", "dg", "db", "dS0"):
        np.testing.assert_allclose(r[key], r2[key], rtol=0, atol=0)
