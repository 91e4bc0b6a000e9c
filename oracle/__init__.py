"""fp64 CPU oracle for the gated delta rule forward -- TEST INFRASTRUCTURE.

Only tests/, the smoke check and the benchmark's CPU-baseline leg import this
package.  The product library never calls it, and it shares no code with the
CUDA path.  The arithmetic lives in gdr_oracle.c (plain C, double precision,
one sequential recurrence per sequence-head, threaded over heads); this module
only marshals arrays.

Every oracle function is pinned by independent checks in tests/test_oracle_pins.py
(chunkwise rederivation, tied-gate reductions, closed forms for beta = 0, exact
recall, the linear-attention special case, exact rational arithmetic on tiny
inputs, decode/forward equivalence); the backward (bwd) in tests/test_oracle_bwd_pins.py
(central finite differences in every mode, closed forms for linear attention and for
a pure decay).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "libgdr_oracle.so")
_MODE = {"gdn2": 0, "kda": 1, "gdn": 2, "bonly": 3, "wonly": 4}
_lib = None


def build(force: bool = False) -> str:
    """Compile gdr_oracle.c with gcc into oracle/libgdr_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdr_oracle_fwd.argtypes = [dp] * 9 + [ctypes.c_int] * 7
        lib.gdr_oracle_fwd.restype = ctypes.c_int
        lib.gdr_oracle_decode.argtypes = [dp] * 8 + [ctypes.c_int] * 6
        lib.gdr_oracle_decode.restype = ctypes.c_int
        lib.gdr_oracle_bwd.argtypes = [dp] * 16 + [ctypes.c_int] * 7
        lib.gdr_oracle_bwd.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    """Exact upcast of a torch tensor / numpy array (fp32 or bf16) to fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def fwd(q, k, v, g, b, w=None, S0=None, mode="gdn2", nthreads=None):
    """Sequential fp64 recurrence over [B,H,T].  Returns (o [B,H,T,dv], S_T [B,H,dk,dv])."""
    lib = _load()
    q, k, v, g, b, w, S0 = map(_f64, (q, k, v, g, b, w, S0))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = lib.gdr_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0),
                            _ptr(o), _ptr(ST), B, H, T, dk, dv, _MODE[mode],
                            nthreads or default_threads())
    if rc != 0:
        raise ValueError("gdr_oracle_fwd: bad arguments")
    return o, ST


def decode(q, k, v, g, b, w=None, S=None, mode="gdn2", nthreads=None):
    """One-token step.  q,k [N,H,dk]; v [N,H,dv]; g [N,H,dk] (gdn: [N,H]);
    b [N,H,dk] (kda/gdn: beta [N,H]; wonly: [N,H]); w [N,H,dv] (bonly: [N,H]);
    S [N,H,dk,dv].  Returns (o, S_new)."""
    lib = _load()
    q, k, v, g, b, w = map(_f64, (q, k, v, g, b, w))
    S = np.array(_f64(S), copy=True)
    N, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((N, H, dv))
    rc = lib.gdr_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S),
                               _ptr(o), N, H, dk, dv, _MODE[mode], nthreads or default_threads())
    if rc != 0:
        raise ValueError("gdr_oracle_decode: bad arguments")
    return o, S


def bwd(q, k, v, g, b, w=None, S0=None, dO=None, dST=None, mode="gdn2", nthreads=None):
    """Gradient of L = sum(o * dO) + sum(S_T * dST) with respect to every input of fwd
    (adjoint of the sequential recurrence, gdr_oracle_bwd).  Returns a dict with dq, dk,
    dv, dg, db, dw (None when the mode has no w) and dS0, each shaped like its input
    (dS0 like S0, [B,H,dk,dv], also when S0 is None)."""
    lib = _load()
    q, k, v, g, b, w, S0, dO, dST = map(_f64, (q, k, v, g, b, w, S0, dO, dST))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dg=np.zeros_like(g),
               db=np.zeros_like(b), dw=None if w is None else np.zeros_like(w),
               dS0=np.zeros((B, H, dk, dv)))
    rc = lib.gdr_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                            _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                            _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]), B, H, T, dk, dv,
                            _MODE[mode], nthreads or default_threads())
    if rc != 0:
        raise ValueError("gdr_oracle_bwd: bad arguments")
    return out


def fwd_heads(inp, heads, nthreads=None):
    """Oracle on a sample of (b, h) pairs of a workload's inputs (dict from
    workload.make_inputs).  Returns (o [n,T,dv], S_T [n,dk,dv]) in the order of
    `heads`; each sequence-head is independent, so this equals slicing the full
    oracle result."""
    def pick(x):
        if x is None:
            return None
        return np.stack([_f64(x[b_, h_]) for (b_, h_) in heads])[:, None]
    o, ST = fwd(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["g"]), pick(inp["b"]),
                pick(inp["w"]), pick(inp["S0"]), mode=inp["mode"], nthreads=nthreads)
    return o[:, 0], ST[:, 0]
