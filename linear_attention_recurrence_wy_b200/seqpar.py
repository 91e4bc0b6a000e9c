"""Sequence split across GPUs: one state hand-off per segment, over torch.distributed.

Only the state crosses chunk borders (Gated DeltaNet-2 Review §3-2.5, "Chunkwise WY
training"), and the recurrence is affine in it: over a segment, S_end = M S_start + S_local
(Gated DeltaNet-2 Q&A page, Q3 update equation).  Each of R ranks holds one contiguous
range of the tokens of every sequence-head, in rank order, and

  1. computes its segment's maps on its GPU: S_local, the end state reached from the
     sequence's S0 (rank 0) or from zero (the others), and -- ranks 1 .. R-2, the only ones
     whose map anyone needs -- M, the end state reached from the identity with the write
     term dropped (gdr_chunk_fwd_segment_maps);
  2. exchanges them: one all-gather of S_local (and one of M when R > 2), 64 KB per
     sequence-head each, over NCCL (NVLink) -- the only collective on the path;
  3. chains them to its own start state in fp32 (gdr_chain_segment_states):
     S_start(0) = S0, S_start(1) = S_local(0), S_start(r+1) = M(r) S_start(r) + S_local(r);
  4. runs the forward on its range from that state (gdr_chunk_fwd).

Rank r owns o of its token range; the last rank's end state is S_T (every other rank's end
state equals the next rank's start state).  Every rank takes the same collective steps in
the same order.  The compute steps go through `ops` (the library by default), so the
exchange and chaining logic runs unchanged with other implementations of the three steps.
"""
from __future__ import annotations

import torch


class LibraryOps:
    """The three compute steps of a rank, on its GPU through libgdr."""

    def maps(self, q, k, v, g, b, w, S0, want_M, mode, chunk):
        from . import segment_maps
        return segment_maps(q, k, v, g, b, w, S0, mode=mode, chunk=chunk, want_M=want_M)

    def chain(self, M_all, S_local_all, S0, r):
        from . import chain_segment_states
        return chain_segment_states(M_all, S_local_all, S0, r)

    def fwd(self, q, k, v, g, b, w, S_start, mode, chunk):
        from . import chunk_fwd
        return chunk_fwd(q, k, v, g, b, w, S_start, mode=mode, chunk=chunk)


def _all_gather(x, group):
    import torch.distributed as dist
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def chunk_fwd_seqpar(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, group=None, ops=None):
    """The forward of a sequence split across the ranks of `group` (see the module note).
    q, k, v, g, b, w: this rank's token range of every sequence-head, [B,H,T_r,.] (ranks in
    sequence order); S0: the sequence's start state, read on rank 0 only.  Returns
    (o of this rank's range, this rank's end state -- S_T on the last rank)."""
    import torch.distributed as dist
    ops = ops if ops is not None else LibraryOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    want_M = 0 < rank < world - 1
    S_local, M = ops.maps(q, k, v, g, b, w, S0 if rank == 0 else None, want_M, mode, chunk)
    S_all = _all_gather(S_local, group)
    M_all = None
    if world > 2:
        if M is None:
            dk = q.shape[-1]
            M = torch.zeros(*S_local.shape[:-2], dk, dk, dtype=S_local.dtype, device=S_local.device)
        M_all = _all_gather(M, group)
    S_start = ops.chain(M_all, S_all, S0 if rank == 0 else None, rank)
    return ops.fwd(q, k, v, g, b, w, S_start, mode, chunk)
