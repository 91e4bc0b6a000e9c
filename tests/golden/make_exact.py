"""Write exact_tiny.json: tiny worked examples computed in exact rational arithmetic.

The pages print no numeric worked example, so this fixture is derived from the
update equation itself (Gated DeltaNet-2 Q&A page, Q3; Gated DeltaNet-2 Review
§3-1), evaluated as explicit matrix products over Python Fractions:

    S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T,   o_t = S_t^T q_t

with D_t = diag(a_t) for rational decay factors a_t; the stored g_log is the
double nearest to log(a_t).  Inputs are small dyadic rationals, so they are
exact in binary floating point.  This script calls neither the oracle nor the
CUDA library; rerun it with `python tests/golden/make_exact.py`.
"""
from __future__ import annotations

import json
import math
import os
import random
from fractions import Fraction as F

HERE = os.path.dirname(os.path.abspath(__file__))


def matmul(A, B):
    return [[sum(A[i][t] * B[t][j] for t in range(len(B))) for j in range(len(B[0]))]
            for i in range(len(A))]


def add(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def outer(x, y):
    return [[xi * yj for yj in y] for xi in x]


def eye(n):
    return [[F(int(i == j)) for j in range(n)] for i in range(n)]


def diag(x):
    return [[x[i] if i == j else F(0) for j in range(len(x))] for i in range(len(x))]


def run_exact(q, k, v, a, b, w, S0):
    dk, dv = len(k[0]), len(v[0])
    S = [row[:] for row in S0]
    outs = []
    for t in range(len(q)):
        bk = [b[t][i] * k[t][i] for i in range(dk)]
        erase = add(eye(dk), [[-x for x in row] for row in outer(k[t], bk)])
        wv = [w[t][j] * v[t][j] for j in range(dv)]
        S = add(matmul(matmul(erase, diag(a[t])), S), outer(k[t], wv))
        outs.append([sum(S[i][j] * q[t][i] for i in range(dk)) for j in range(dv)])
    return outs, S


def dyadic(rng, lo=-8, hi=8, den=8):
    return F(rng.randint(lo, hi), den)


def case(seed, T, dk, dv, tied=None):
    rng = random.Random(seed)
    q = [[dyadic(rng) for _ in range(dk)] for _ in range(T)]
    k = [[dyadic(rng) for _ in range(dk)] for _ in range(T)]
    v = [[dyadic(rng) for _ in range(dv)] for _ in range(T)]
    choices = [F(1, 2), F(3, 4), F(7, 8), F(1, 1), F(1, 4)]
    if tied == "gdn":
        a = [[rng.choice(choices)] * dk for _ in range(T)]
    else:
        a = [[rng.choice(choices) for _ in range(dk)] for _ in range(T)]
    if tied is None:
        b = [[F(rng.randint(0, 8), 8) for _ in range(dk)] for _ in range(T)]
        w = [[F(rng.randint(0, 8), 8) for _ in range(dv)] for _ in range(T)]
    else:
        beta = [F(rng.randint(0, 8), 8) for _ in range(T)]
        b = [[beta[t]] * dk for t in range(T)]
        w = [[beta[t]] * dv for t in range(T)]
    S0 = [[dyadic(rng, den=4) for _ in range(dv)] for _ in range(dk)]
    o, ST = run_exact(q, k, v, a, b, w, S0)
    fl = lambda M: [[float(x) for x in row] for row in M]
    rec = dict(seed=seed, T=T, dk=dk, dv=dv, mode=tied or "gdn2",
               q=fl(q), k=fl(k), v=fl(v),
               g=[[math.log(x) for x in row] for row in a],
               S0=fl(S0), o=fl(o), ST=fl(ST))
    if tied is None:
        rec["b"], rec["w"] = fl(b), fl(w)
    else:
        rec["beta"] = [float(x[0]) for x in b]
    if tied == "gdn":
        rec["g"] = [row[0] for row in rec["g"]]
    return rec


def main():
    cases = [case(1, 3, 2, 3), case(2, 4, 3, 2), case(3, 4, 2, 2, tied="kda"),
             case(4, 3, 3, 3, tied="gdn")]
    doc = {
        "source": "Gated DeltaNet-2 Q&A page, Q3 update equation; Gated DeltaNet-2 Review "
                  "section 3-1; tied reductions per the same Q3 and the Gated DeltaNet "
                  "explainer's mechanism section. Exact Fraction arithmetic of the matrix "
                  "form; g = log(decay factor) rounded to double.",
        "generator": "tests/golden/make_exact.py",
        "cases": cases,
    }
    with open(os.path.join(HERE, "exact_tiny.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
