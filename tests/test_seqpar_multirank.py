"""The sequence split across GPUs (linear_attention_recurrence_wy_b200.seqpar), its rank
roles, exchange and chaining, on CPU with gloo (world sizes 2 and 3).

Each rank holds one contiguous token range of every sequence-head.  The three compute steps
of a rank (its segment's maps, the chaining of the gathered maps, the forward from its
start state) run here as plain per-token CPU stand-ins in float64 -- the transition map is
the product of the per-token matrices (I - k (b.k)^T) diag(exp g) -- while the product's
orchestration decides who computes what, exchanges the maps by all-gather and hands them on.
The oracle is only the checker: every rank's output range, the start state it received and
the last rank's end state must equal the whole-sequence oracle."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workload
from linear_attention_recurrence_wy_b200 import seqpar


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gates(q, k, v, g, b, w, mode, i, t):
    """Per-token vectors of sequence-head i at token t: k, q, v, e^g [dk], b [dk], w [dv]."""
    dk, dv = q.shape[-1], v.shape[-1]
    kt, qt, vt = k[i, t], q[i, t], v[i, t]
    eg = np.exp(g[i, t]) if g.ndim == 3 else np.full(dk, np.exp(g[i, t]))
    bt = b[i, t] if b.ndim == 3 else np.full(dk, b[i, t])
    if w is None:                       # tied modes: the write gate is beta
        wt = np.full(dv, b[i, t])
    else:
        wt = w[i, t] if w.ndim == 3 else np.full(dv, w[i, t])
    return kt, qt, vt, eg, bt, wt


class CpuOps:
    """Plain per-token float64 stand-ins of the three compute steps (tensors [B,H,T,.])."""

    def __init__(self):
        self.S_start = None

    @staticmethod
    def _flat(*xs):
        out = []
        for x in xs:
            if x is None:
                out.append(None)
            else:
                a = x.double().numpy()
                out.append(a.reshape(-1, *a.shape[2:]))
        return out

    def maps(self, q, k, v, g, b, w, S0, want_M, mode, chunk):
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        q_, k_, v_, g_, b_, w_ = self._flat(q, k, v, g, b, w)
        S = np.zeros((B * H, dk, dv)) if S0 is None else S0.double().numpy().reshape(B * H, dk, dv).copy()
        M = np.tile(np.eye(dk), (B * H, 1, 1))
        for i in range(B * H):
            for t in range(T):
                kt, qt, vt, eg, bt, wt = _gates(q_, k_, v_, g_, b_, w_, mode, i, t)
                A = (np.eye(dk) - np.outer(kt, bt * kt)) * eg[None, :]   # (I - k (b.k)^T) diag(e^g)
                S[i] = A @ S[i] + np.outer(kt, wt * vt)
                M[i] = A @ M[i]
        to = lambda a, s: torch.from_numpy(a.reshape(s))
        return to(S, (B, H, dk, dv)), (to(M, (B, H, dk, dk)) if want_M else None)

    def chain(self, M_all, S_all, S0, r):
        R, B, H, dk, dv = S_all.shape
        if r == 0:
            S = torch.zeros(B, H, dk, dv, dtype=torch.float64) if S0 is None else S0.double()
        else:
            S = S_all[0].double()
            for i in range(1, r):
                S = M_all[i].double() @ S + S_all[i].double()
        self.S_start = S
        return S

    def fwd(self, q, k, v, g, b, w, S_start, mode, chunk):
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        q_, k_, v_, g_, b_, w_ = self._flat(q, k, v, g, b, w)
        S = S_start.double().numpy().reshape(B * H, dk, dv).copy()
        o = np.zeros((B * H, T, dv))
        for i in range(B * H):
            for t in range(T):
                kt, qt, vt, eg, bt, wt = _gates(q_, k_, v_, g_, b_, w_, mode, i, t)
                S[i] = eg[:, None] * S[i]
                S[i] = S[i] + np.outer(kt, wt * vt - S[i].T @ (bt * kt))
                o[i, t] = S[i].T @ qt
        return torch.from_numpy(o.reshape(B, H, T, dv)), torch.from_numpy(S.reshape(B, H, dk, dv))


def _worker(rank, world, port, mode, T, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        d = workload.make_small(2, 2, T, 16, 16, mode=mode, dtype="f32", seed=40 + world, g_scale=0.5,
                                s0_std=0.1)
        cuts = [T * r // world for r in range(world + 1)]
        lo, hi = cuts[rank], cuts[rank + 1]
        sl = lambda x: None if x is None else x[:, :, lo:hi].contiguous()
        ops = CpuOps()
        o, S_end = seqpar.chunk_fwd_seqpar(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["b"]),
                                           sl(d["w"]), d["S0"] if rank == 0 else None, mode=mode, ops=ops)
        # the checker: the oracle on the whole sequence, and on the prefix before this range
        o_ref, S_ref = oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode)
        pre = lambda x: None if x is None else x[:, :, :lo].contiguous()
        if lo > 0:
            _, S_lo = oracle.fwd(pre(d["q"]), pre(d["k"]), pre(d["v"]), pre(d["g"]), pre(d["b"]), pre(d["w"]),
                                 d["S0"], mode=mode)
        else:
            S_lo = d["S0"].double().numpy()
        out[rank] = dict(o_err=float(np.abs(o.numpy() - o_ref[:, :, lo:hi]).max()),
                         start_err=float(np.abs(ops.S_start.numpy() - S_lo).max()),
                         end_err=float(np.abs(S_end.numpy() - S_ref).max()) if rank == world - 1 else 0.0,
                         tokens=(lo, hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mode", [(2, "gdn2"), (3, "gdn2"), (3, "kda")])
def test_split_across_ranks_matches_the_whole_sequence(world, mode):
    T = 45   # uneven ranges: 22/23 or 15/15/15 tokens
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), mode, T, out), nprocs=world, join=True)
    covered = []
    for r in range(world):
        res = out[r]
        covered.append(res["tokens"])
        assert res["o_err"] < 1e-9, (r, res)
        assert res["start_err"] < 1e-9, (r, res)
        assert res["end_err"] < 1e-9, (r, res)
    assert covered[0][0] == 0 and covered[-1][1] == T
    assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))


class _RecordingOps(CpuOps):
    def __init__(self):
        super().__init__()
        self.want = None

    def maps(self, q, k, v, g, b, w, S0, want_M, mode, chunk):
        self.want = (want_M, S0 is not None)
        return super().maps(q, k, v, g, b, w, S0, want_M, mode, chunk)


def _roles_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        d = workload.make_small(1, 1, 8, 4, 4, mode="gdn2", dtype="f32", seed=3, s0_std=0.1)
        ops = _RecordingOps()
        seqpar.chunk_fwd_seqpar(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode="gdn2", ops=ops)
        out[rank] = ops.want
    finally:
        dist.destroy_process_group()


def test_only_inner_ranks_compute_a_transition_map_and_only_rank_0_reads_S0():
    world = 4
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_roles_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert [out[r] for r in range(world)] == [(False, True), (True, False), (True, False), (False, False)]
