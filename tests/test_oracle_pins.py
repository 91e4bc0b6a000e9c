"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test targets a different plausible mistake (dropped term, wrong sign,
swapped gate, transposed state, decay on the wrong side of the erase, read-out
from the pre-update state, wrong tied reduction).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import chunk_ref
import workload

GOLD = os.path.join(os.path.dirname(__file__), "golden", "exact_tiny.json")


def rnd_inputs(seed, B, H, T, dk, dv, mode="gdn2", g_scale=1.0, s0=True):
    d = workload.make_small(B, H, T, dk, dv, mode=mode, dtype="f32", seed=seed,
                            g_scale=g_scale, s0_std=0.3 if s0 else 0.0)
    return d


def run_oracle(d, **kw):
    return oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=d["mode"], **kw)


# 1. exact rational worked examples of the matrix form of the update equation
def test_exact_rational_examples():
    doc = json.load(open(GOLD))
    for c in doc["cases"]:
        q = np.array(c["q"])[None, None]
        k = np.array(c["k"])[None, None]
        v = np.array(c["v"])[None, None]
        g = np.array(c["g"])[None, None]
        S0 = np.array(c["S0"])[None, None]
        if c["mode"] == "gdn2":
            b, w = np.array(c["b"])[None, None], np.array(c["w"])[None, None]
        else:
            b, w = np.array(c["beta"])[None, None], None
        o, ST = oracle.fwd(q, k, v, g, b, w, S0, mode=c["mode"], nthreads=1)
        np.testing.assert_allclose(o[0, 0], np.array(c["o"]), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ST[0, 0], np.array(c["ST"]), rtol=1e-12, atol=1e-13)


# 2. chunkwise WY rederivation agrees with the sequential recurrence
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 17, 64, 65, 130])
def test_chunkwise_rederivation(mode, C, T):
    d = rnd_inputs(10 + T + C, 2, 2, T, 16, 24, mode=mode, g_scale=0.5)
    o, ST = run_oracle(d, nthreads=2)
    o2, ST2 = chunk_ref.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                  mode=mode, C=C)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(ST, ST2, rtol=1e-10, atol=1e-11)


# 3. tied reductions: GDN-2 with b = w = beta*1 is KDA; KDA with a scalar decay is GDN;
#    GDN equals alpha (I - beta k k^T) S + beta k v^T written as matrices.
def test_tied_reductions():
    d = rnd_inputs(3, 2, 2, 40, 8, 6, mode="kda")
    dk, dv = 8, 6
    beta = d["b"].double().numpy()
    o_kda, S_kda = run_oracle(d)
    b_full = np.repeat(beta[..., None], dk, -1)
    w_full = np.repeat(beta[..., None], dv, -1)
    o_g2, S_g2 = oracle.fwd(d["q"], d["k"], d["v"], d["g"], b_full, w_full, d["S0"], mode="gdn2")
    np.testing.assert_allclose(o_kda, o_g2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_kda, S_g2, rtol=1e-13, atol=1e-14)

    gs = d["g"][..., 0].clone()                   # one scalar decay per token
    o_gdn, S_gdn = oracle.fwd(d["q"], d["k"], d["v"], gs, d["b"], None, d["S0"], mode="gdn")
    g_full = gs[..., None].expand(-1, -1, -1, dk)
    o_k2, S_k2 = oracle.fwd(d["q"], d["k"], d["v"], g_full, d["b"], None, d["S0"], mode="kda")
    np.testing.assert_allclose(o_gdn, o_k2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_gdn, S_k2, rtol=1e-13, atol=1e-14)

    # the Gated DeltaNet explainer's form, as explicit matrices
    q, k, v = (d[x].double().numpy() for x in ("q", "k", "v"))
    alpha = np.exp(gs.double().numpy())
    for bi in range(2):
        for hi in range(2):
            S = d["S0"][bi, hi].double().numpy().copy()
            for t in range(40):
                kt, vt, qt = k[bi, hi, t], v[bi, hi, t], q[bi, hi, t]
                bt, at = beta[bi, hi, t], alpha[bi, hi, t]
                S = at * (np.eye(dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, vt)
                np.testing.assert_allclose(o_gdn[bi, hi, t], S.T @ qt, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(S_gdn[bi, hi], S, rtol=1e-11, atol=1e-12)


# 3b. gate-ablation variants (Gated DeltaNet-2 Review §5, "Gate ablation"): b-only is
#     GDN-2 with the write gate w_t * 1, w-only is GDN-2 with the erase gate b_t * 1; the
#     expanded erase range b in [0, 2] keeps the chunkwise form exact.
def test_gate_ablation_variants():
    dk, dv = 8, 6
    d = rnd_inputs(31, 2, 2, 37, dk, dv, mode="bonly")
    w_full = np.repeat(d["w"].double().numpy()[..., None], dv, -1)
    o1, S1 = run_oracle(d)
    o2, S2 = oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], w_full, d["S0"], mode="gdn2")
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S1, S2, rtol=1e-13, atol=1e-14)
    # a write gate that varies over channels must matter: the scalar is not a channel read
    w_ch = w_full.copy()
    w_ch[..., 0] *= 0.5
    o3, _ = oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], w_ch, d["S0"], mode="gdn2")
    assert np.max(np.abs(o3 - o1)) > 1e-3

    d = rnd_inputs(32, 2, 2, 37, dk, dv, mode="wonly")
    b_full = np.repeat(d["b"].double().numpy()[..., None], dk, -1)
    o1, S1 = run_oracle(d)
    o2, S2 = oracle.fwd(d["q"], d["k"], d["v"], d["g"], b_full, d["w"], d["S0"], mode="gdn2")
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S1, S2, rtol=1e-13, atol=1e-14)

    d = workload.make_small(2, 2, 70, 12, 10, mode="gdn2", dtype="f32", seed=33, g_scale=0.5,
                            s0_std=0.3, b_range=2.0)
    assert float(d["b"].max()) > 1.0                  # the expanded range is in use
    o, ST = run_oracle(d)
    o2, ST2 = chunk_ref.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                  mode="gdn2", C=32)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(ST, ST2, rtol=1e-10, atol=1e-11)


# 4. beta = 0: nothing is erased or written; the state only decays (closed form)
def test_zero_gates_pure_decay():
    d = rnd_inputs(4, 2, 3, 50, 12, 10, g_scale=0.3)
    d["b"] = torch.zeros_like(d["b"])
    d["w"] = torch.zeros_like(d["w"])
    o, ST = run_oracle(d)
    g = d["g"].double().numpy()
    S0 = d["S0"].double().numpy()
    q = d["q"].double().numpy()
    cum = np.cumsum(g, axis=2)                                   # [B,H,T,dk]
    ST_ref = np.exp(cum[:, :, -1])[..., None] * S0
    o_ref = np.einsum("bhtd,bhdv->bhtv", q * np.exp(cum), S0)
    np.testing.assert_allclose(ST, ST_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)


# 5. exact recall: orthonormal keys, no decay, b = 1 -> S_T^T k_j = w_j . v_j
@pytest.mark.parametrize("unit_w", [True, False])
def test_exact_recall_orthonormal_keys(unit_w):
    rng = np.random.default_rng(5)
    dk, dv = 16, 9
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[None, None]                                          # T = dk orthonormal keys
    v = rng.standard_normal((1, 1, dk, dv))
    q = rng.standard_normal((1, 1, dk, dk))
    g = np.zeros((1, 1, dk, dk))
    b = np.ones((1, 1, dk, dk))
    w = np.ones((1, 1, dk, dv)) if unit_w else rng.uniform(0, 1, (1, 1, dk, dv))
    S0 = rng.standard_normal((1, 1, dk, dv))
    _, ST = oracle.fwd(q, k, v, g, b, w, S0, mode="gdn2")
    recalled = k[0, 0] @ ST[0, 0]                                 # row j = S_T^T k_j
    np.testing.assert_allclose(recalled, w[0, 0] * v[0, 0], rtol=1e-12, atol=1e-12)


# 6. g = 0, b = 0, w = 1 is causal linear attention
def test_linear_attention_special_case():
    d = rnd_inputs(6, 1, 2, 33, 7, 5)
    d["g"] = torch.zeros_like(d["g"])
    d["b"] = torch.zeros_like(d["b"])
    d["w"] = torch.ones_like(d["w"])
    o, ST = run_oracle(d)
    q, k, v, S0 = (d[x].double().numpy() for x in ("q", "k", "v", "S0"))
    scores = np.einsum("bhtd,bhsd->bhts", q, k) * np.tril(np.ones((33, 33)))
    o_ref = np.einsum("bhtd,bhdv->bhtv", q, S0) + scores @ v
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST, S0 + np.einsum("bhtd,bhtv->bhdv", k, v), rtol=1e-12, atol=1e-12)


# 7. brute force with explicit dk x dk transition matrices, tiny shapes
def test_bruteforce_matrix_form():
    d = rnd_inputs(7, 1, 1, 4, 2, 2)
    o, ST = run_oracle(d)
    q, k, v, g, b, w, S0 = (d[x][0, 0].double().numpy() for x in ("q", "k", "v", "g", "b", "w", "S0"))
    S = S0.copy()
    for t in range(4):
        M = (np.eye(2) - np.outer(k[t], b[t] * k[t])) @ np.diag(np.exp(g[t]))
        S = M @ S + np.outer(k[t], w[t] * v[t])
        np.testing.assert_allclose(o[0, 0, t], S.T @ q[t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ST[0, 0], S, rtol=1e-13, atol=1e-14)


# 8. the decode step repeated T times equals the forward; state hand-off is exact
@pytest.mark.parametrize("mode", ["gdn2", "kda", "gdn", "bonly", "wonly"])
def test_decode_steps_equal_forward_and_split(mode):
    d = rnd_inputs(8, 2, 2, 21, 8, 8, mode=mode)
    o, ST = run_oracle(d)
    S = d["S0"].double().numpy()
    for t in range(21):
        sl = lambda x: None if x is None else x[:, :, t]
        od, S = oracle.decode(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["b"]),
                              sl(d["w"]), S, mode=mode)
        np.testing.assert_allclose(od, o[:, :, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, ST, rtol=1e-12, atol=1e-13)

    cut = 13
    part = lambda x, s: None if x is None else x[:, :, s]
    o1, S1 = oracle.fwd(*(part(d[x], slice(0, cut)) for x in ("q", "k", "v", "g", "b", "w")),
                        d["S0"], mode=mode)
    o2, S2 = oracle.fwd(*(part(d[x], slice(cut, None)) for x in ("q", "k", "v", "g", "b", "w")),
                        S1, mode=mode)
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, ST, rtol=1e-12, atol=1e-13)


def test_empty_sequence_returns_initial_state():
    d = rnd_inputs(9, 1, 2, 0, 4, 4)
    o, ST = run_oracle(d)
    assert o.shape == (1, 2, 0, 4)
    np.testing.assert_array_equal(ST, d["S0"].double().numpy())


def test_threads_do_not_change_result():
    d = rnd_inputs(11, 3, 3, 20, 8, 8)
    o1, S1 = run_oracle(d, nthreads=1)
    o4, S4 = run_oracle(d, nthreads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(S1, S4)
