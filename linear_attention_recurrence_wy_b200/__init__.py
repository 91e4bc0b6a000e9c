"""Gated delta rule forward on NVIDIA B200 (sm_100a): thin Python binding of libgdr.

The arithmetic runs in libgdr.so's CUDA kernels; this module only checks tensor
shapes and dtypes, allocates outputs with PyTorch and passes raw device pointers
and the current CUDA stream to the C ABI (include/gdr.h).  There is no CPU or
PyTorch fallback: if libgdr.so is missing or a call fails, an exception is raised.

Raw C-ABI names (integer pointers):  gdr_chunk_fwd, gdr_chunk_fwd_split,
gdr_chunk_fwd_split_noalloc, gdr_chunk_fwd_split_segments, gdr_chunk_fwd_split_workspace,
gdr_chunk_fwd_two_phase, gdr_chunk_fwd_two_phase_segments, gdr_chunk_fwd_two_phase_workspace,
gdr_mixer_fwd, gdr_chunk_bwd, gdr_chunk_bwd_workspace, gdr_decode_step,
gdr_chunk_fwd_segment_maps, gdr_chain_segment_states, gdr_last_device_error,
gdr_status_string, gdr_test_set_first_wait_limit, gdr_debug_build, gdr_debug_bounds_site.
Tensor wrappers:  chunk_fwd, chunk_fwd_split, chunk_fwd_two_phase, chunk_fwd_auto, chunk_fwd_host, mixer_fwd, mixer_fwd_host,
chunk_bwd, decode_step, segment_maps, chain_segment_states; the sequence split across GPUs
(torch.distributed): seqpar.chunk_fwd_seqpar.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# GDR_DEBUG=1 loads the debug build (in-kernel bounds checks, build.py --debug) instead
LIB_PATH = os.path.join(_PKG, "libgdr_debug.so" if os.environ.get("GDR_DEBUG") == "1" else "libgdr.so")
MODES = {"gdn2": 0, "kda": 1, "gdn": 2, "bonly": 3, "wonly": 4}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
LAYOUTS = {"bhtd": 0, "bthd": 1}
_lib = None


class GdrError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {gdr_status_string(code)} ({code})")


def lib():
    """Load libgdr.so (built in-tree by build.py; libgdr_debug.so when GDR_DEBUG=1); raises if
    it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{os.path.basename(LIB_PATH)} not built: run python -m "
                              f"linear_attention_recurrence_wy_b200.build (expected at {LIB_PATH})")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        L.gdr_chunk_fwd.argtypes = [vp] * 9 + [ci] * 8 + [vp]
        L.gdr_chunk_fwd.restype = ci
        L.gdr_chunk_fwd_split.argtypes = [vp] * 9 + [ci] * 9 + [vp, ctypes.c_ulonglong, vp]
        L.gdr_chunk_fwd_split.restype = ci
        L.gdr_chunk_fwd_split_noalloc.argtypes = [vp] * 9 + [ci] * 9 + [vp]
        L.gdr_chunk_fwd_split_noalloc.restype = ci
        L.gdr_chunk_fwd_split_segments.argtypes = [ci] * 7
        L.gdr_chunk_fwd_split_segments.restype = ci
        L.gdr_chunk_fwd_split_workspace.argtypes = [ci] * 5
        L.gdr_chunk_fwd_split_workspace.restype = ctypes.c_ulonglong
        L.gdr_chunk_fwd_two_phase.argtypes = [vp] * 9 + [ci] * 9 + [vp, ctypes.c_ulonglong, vp]
        L.gdr_chunk_fwd_two_phase.restype = ci
        L.gdr_chunk_fwd_two_phase_segments.argtypes = [ci] * 7
        L.gdr_chunk_fwd_two_phase_segments.restype = ci
        L.gdr_chunk_fwd_two_phase_workspace.argtypes = [ci] * 7
        L.gdr_chunk_fwd_two_phase_workspace.restype = ctypes.c_ulonglong
        L.gdr_mixer_fwd.argtypes = [vp] * 11 + [ci] * 9 + [ctypes.c_float] * 2 + [vp]
        L.gdr_mixer_fwd.restype = ci
        L.gdr_chunk_bwd.argtypes = [vp] * 16 + [ci] * 7 + [vp, ctypes.c_ulonglong, vp]
        L.gdr_chunk_bwd.restype = ci
        L.gdr_chunk_bwd_workspace.argtypes = [ci] * 5
        L.gdr_chunk_bwd_workspace.restype = ctypes.c_ulonglong
        L.gdr_decode_step.argtypes = [vp] * 8 + [ci] * 6 + [vp]
        L.gdr_decode_step.restype = ci
        L.gdr_last_device_error.argtypes = [vp]
        L.gdr_last_device_error.restype = ci
        L.gdr_chunk_fwd_segment_maps.argtypes = [vp] * 9 + [ci] * 8 + [vp]
        L.gdr_chunk_fwd_segment_maps.restype = ci
        L.gdr_chain_segment_states.argtypes = [vp] * 4 + [ci] * 6 + [vp]
        L.gdr_chain_segment_states.restype = ci
        L.gdr_debug_build.argtypes = []
        L.gdr_debug_build.restype = ci
        L.gdr_debug_bounds_site.argtypes = []
        L.gdr_debug_bounds_site.restype = ci
        L.gdr_test_set_first_wait_limit.argtypes = [ctypes.c_uint]
        L.gdr_test_set_first_wait_limit.restype = None
        L.gdr_status_string.argtypes = [ci]
        L.gdr_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ---- raw C-ABI names -------------------------------------------------------------------
def gdr_chunk_fwd(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype, stream):
    return lib().gdr_chunk_fwd(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                               dtype, stream)


def gdr_chunk_fwd_split(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype, nseg,
                        workspace, workspace_bytes, stream):
    return lib().gdr_chunk_fwd_split(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                                     dtype, nseg, workspace, workspace_bytes, stream)


def gdr_chunk_fwd_split_noalloc(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                                dtype, nseg, stream):
    return lib().gdr_chunk_fwd_split_noalloc(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv,
                                             chunk, mode, dtype, nseg, stream)


def gdr_chunk_fwd_split_segments(B, H, T, dk, dv, chunk, dtype):
    return lib().gdr_chunk_fwd_split_segments(B, H, T, dk, dv, chunk, dtype)


def gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg):
    return lib().gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg)


def gdr_chunk_fwd_two_phase(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype, nseg,
                            workspace, workspace_bytes, stream):
    return lib().gdr_chunk_fwd_two_phase(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                                         dtype, nseg, workspace, workspace_bytes, stream)


def gdr_chunk_fwd_two_phase_segments(B, H, T, dk, dv, chunk, dtype):
    return lib().gdr_chunk_fwd_two_phase_segments(B, H, T, dk, dv, chunk, dtype)


def gdr_chunk_fwd_two_phase_workspace(B, H, T, dk, dv, chunk, nseg):
    return lib().gdr_chunk_fwd_two_phase_workspace(B, H, T, dk, dv, chunk, nseg)


def gdr_mixer_fwd(q, k, v, xg, xb, xw, z, norm_weight, S0, y, S_T, B, H, T, dk, dv, chunk, mode,
                  dtype, layout, b_range, eps, stream):
    return lib().gdr_mixer_fwd(q, k, v, xg, xb, xw, z, norm_weight, S0, y, S_T, B, H, T, dk, dv,
                               chunk, mode, dtype, layout, b_range, eps, stream)


def gdr_chunk_bwd(q, k, v, g_log, b, w, S0, dO, dS_T, dq, dk_, dv_, dg, db, dw, dS0, B, H, T, dk, dv,
                  mode, dtype, workspace, workspace_bytes, stream):
    return lib().gdr_chunk_bwd(q, k, v, g_log, b, w, S0, dO, dS_T, dq, dk_, dv_, dg, db, dw, dS0, B, H,
                               T, dk, dv, mode, dtype, workspace, workspace_bytes, stream)


def gdr_chunk_bwd_workspace(B, H, T, dk, dv):
    return lib().gdr_chunk_bwd_workspace(B, H, T, dk, dv)


def gdr_decode_step(q, k, v, g_log, b, w, S, o, N, H, dk, dv, mode, dtype, stream):
    return lib().gdr_decode_step(q, k, v, g_log, b, w, S, o, N, H, dk, dv, mode, dtype, stream)


def gdr_last_device_error(stream=None):
    return lib().gdr_last_device_error(stream)


def gdr_chunk_fwd_segment_maps(q, k, v, g_log, b, w, S0, S_local, M, B, H, T, dk, dv, chunk, mode, dtype,
                               stream=None):
    return lib().gdr_chunk_fwd_segment_maps(q, k, v, g_log, b, w, S0, S_local, M, B, H, T, dk, dv, chunk, mode,
                                            dtype, stream)


def gdr_chain_segment_states(M_all, S_local_all, S0, S_start, R, r, B, H, dk, dv, stream=None):
    return lib().gdr_chain_segment_states(M_all, S_local_all, S0, S_start, R, r, B, H, dk, dv, stream)


def segment_maps(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, want_M=False):
    """Maps of one segment of the sequence held on its own (gdr_chunk_fwd_segment_maps):
    returns (S_local, M) -- the end state reached from S0 (zero if None) and, when want_M,
    the transition map [B,H,dk,dk] (else None).  bf16, dk = dv = 128, chunk 64."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    gshape, bshape, wshape = _gate_shapes(mode, (B, H, T), dk, dv)
    for t, name, shape, tdt in ((q, "q", (B, H, T, dk), dt), (k, "k", (B, H, T, dk), dt),
                                (v, "v", (B, H, T, dv), dt), (g, "g", gshape, torch.float32),
                                (b, "b", bshape, dt)):
        _check(t, name, shape, tdt, dev)
    if wshape is not None:
        _check(w, "w", wshape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    S_local = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    M = torch.empty(B, H, dk, dk, dtype=torch.float32, device=dev) if want_M else None
    rc = gdr_chunk_fwd_segment_maps(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                                    _ptr(w) if wshape is not None else None, _ptr(S0), _ptr(S_local), _ptr(M),
                                    B, H, T, dk, dv, chunk, MODES[mode], DTYPES[dt], _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_segment_maps")
    return S_local, M


def chain_segment_states(M_all, S_local_all, S0, r):
    """Start state of holder r (gdr_chain_segment_states) from the gathered maps
    M_all [R,B,H,dk,dk] (may be None when r < 2) and S_local_all [R,B,H,dk,dv]; S0 is read
    when r = 0 (None: zero)."""
    R, B, H, dk, dv = S_local_all.shape
    dev = S_local_all.device
    _check(S_local_all, "S_local_all", (R, B, H, dk, dv), torch.float32, dev)
    if M_all is not None:
        _check(M_all, "M_all", (R, B, H, dk, dk), torch.float32, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    S_start = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    rc = gdr_chain_segment_states(_ptr(M_all), _ptr(S_local_all), _ptr(S0), _ptr(S_start), R, r, B, H, dk, dv,
                                  _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chain_segment_states")
    return S_start


def gdr_debug_build() -> int:
    return lib().gdr_debug_build()


def gdr_debug_bounds_site() -> int:
    return lib().gdr_debug_bounds_site()


def gdr_test_set_first_wait_limit(polls: int) -> None:
    """Test hook: the first bounded wait of each CTA gives up after `polls` non-blocking
    polls (0 restores the normal bound); see include/gdr.h."""
    lib().gdr_test_set_first_wait_limit(polls)


def gdr_status_string(code: int) -> str:
    return lib().gdr_status_string(int(code)).decode()


# ---- tensor wrappers -------------------------------------------------------------------
def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _check(t, name, shape, dtype, device):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype} != {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


def _gate_shapes(mode, lead, dk, dv):
    """Shapes of g, b and w (None: w unused) for a mode."""
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode!r}")
    if mode == "gdn2":
        return (*lead, dk), (*lead, dk), (*lead, dv)
    if mode == "bonly":
        return (*lead, dk), (*lead, dk), tuple(lead)
    if mode == "wonly":
        return (*lead, dk), tuple(lead), (*lead, dv)
    if mode == "kda":
        return (*lead, dk), tuple(lead), None
    return tuple(lead), tuple(lead), None


def chunk_fwd(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, o=None, S_T=None,
              return_state=True):
    """Chunkwise forward.  q,k [B,H,T,dk], v [B,H,T,dv] (fp32 or bf16, CUDA), g fp32,
    b (beta for kda/gdn, a scalar erase gate for wonly), w (gdn2, bonly: scalar, wonly),
    S0 fp32 [B,H,dk,dv] or None.
    Returns (o, S_T) with S_T None when return_state is False."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    if dt not in DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    gshape, bshape, wshape = _gate_shapes(mode, (B, H, T), dk, dv)
    _check(q, "q", (B, H, T, dk), dt, dev)
    _check(k, "k", (B, H, T, dk), dt, dev)
    _check(v, "v", (B, H, T, dv), dt, dev)
    _check(g, "g", gshape, torch.float32, dev)
    _check(b, "b", bshape, dt, dev)
    if wshape is not None:
        _check(w, "w", wshape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    rc = gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                       _ptr(w) if wshape is not None else None, _ptr(S0), _ptr(o), _ptr(S_T),
                       B, H, T, dk, dv, chunk, MODES[mode], DTYPES[dt], _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd")
    return o, S_T


def chunk_fwd_split(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, nseg=None,
                    workspace=None, o=None, S_T=None, return_state=True):
    """chunk_fwd with each sequence cut into `nseg` segments processed in parallel (for
    long sequences with few sequence-heads).  nseg=None asks the library for its
    recommendation; the workspace (uint8 CUDA tensor) is allocated here when not given."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if nseg is None:
        nseg = gdr_chunk_fwd_split_segments(B, H, T, dk, dv, chunk, DTYPES[dt])
    if nseg <= 1:
        return chunk_fwd(q, k, v, g, b, w, S0, mode=mode, chunk=chunk, o=o, S_T=S_T,
                         return_state=return_state)
    need = gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    gshape, bshape, wshape = _gate_shapes(mode, (B, H, T), dk, dv)
    for t, name, shape, tdt in ((q, "q", (B, H, T, dk), dt), (k, "k", (B, H, T, dk), dt),
                                (v, "v", (B, H, T, dv), dt), (g, "g", gshape, torch.float32),
                                (b, "b", bshape, dt)):
        _check(t, name, shape, tdt, q.device)
    if wshape is not None:
        _check(w, "w", wshape, dt, q.device)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=dt, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    rc = gdr_chunk_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                             _ptr(w) if wshape is not None else None, _ptr(S0), _ptr(o), _ptr(S_T),
                             B, H, T, dk, dv, chunk, MODES[mode], DTYPES[dt], nseg,
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_split")
    return o, S_T


def chunk_fwd_two_phase(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, nseg=None,
                        workspace=None, o=None, S_T=None, return_state=True):
    """chunk_fwd as two phases (gdr_chunk_fwd_two_phase): the WY records of every chunk in
    parallel, then the recurrence over them, its sequences cut into `nseg` segments (None:
    the library's recommendation, at least 1).  The workspace (uint8 CUDA tensor) is
    allocated here when not given.  bf16, dk = dv = 128, chunk 64 only."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    if dt not in DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    if nseg is None:
        nseg = max(1, gdr_chunk_fwd_two_phase_segments(B, H, T, dk, dv, chunk, DTYPES[dt]))
    gshape, bshape, wshape = _gate_shapes(mode, (B, H, T), dk, dv)
    for t, name, shape, tdt in ((q, "q", (B, H, T, dk), dt), (k, "k", (B, H, T, dk), dt),
                                (v, "v", (B, H, T, dv), dt), (g, "g", gshape, torch.float32),
                                (b, "b", bshape, dt)):
        _check(t, name, shape, tdt, dev)
    if wshape is not None:
        _check(w, "w", wshape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    need = gdr_chunk_fwd_two_phase_workspace(B, H, T, dk, dv, chunk, nseg)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    rc = gdr_chunk_fwd_two_phase(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                                 _ptr(w) if wshape is not None else None, _ptr(S0), _ptr(o), _ptr(S_T),
                                 B, H, T, dk, dv, chunk, MODES[mode], DTYPES[dt], nseg,
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_two_phase")
    return o, S_T


def chunk_fwd_auto(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, o=None, S_T=None,
                   return_state=True):
    """chunk_fwd by the path the library expects to be fastest for this problem on this
    device: the two-phase forward, the fused kernel with a sequence split, or the fused
    kernel (workspaces allocated here)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if q.dtype in DTYPES:
        code = DTYPES[q.dtype]
        n2 = gdr_chunk_fwd_two_phase_segments(B, H, T, dk, dv, chunk, code)
        if n2 > 0:
            return chunk_fwd_two_phase(q, k, v, g, b, w, S0, mode=mode, chunk=chunk, nseg=n2, o=o, S_T=S_T,
                                       return_state=return_state)
        if gdr_chunk_fwd_split_segments(B, H, T, dk, dv, chunk, code) > 1:
            return chunk_fwd_split(q, k, v, g, b, w, S0, mode=mode, chunk=chunk, o=o, S_T=S_T,
                                   return_state=return_state)
    return chunk_fwd(q, k, v, g, b, w, S0, mode=mode, chunk=chunk, o=o, S_T=S_T, return_state=return_state)


def _pipelined_host_call(inputs, outputs, groups, run, device):
    """Run `run(lo, hi, dev_inputs, dev_outputs)` on groups [lo, hi) of the leading unit axis
    of host tensors, overlapping the host-to-device copies of group i+1 (a copy stream), the
    library call on group i (the current stream) and the device-to-host copies of group i-1
    (a second copy stream).  inputs / outputs: lists of host tensors (None allowed) viewed
    with the unit axis first; returns nothing (the outputs are filled).  The current stream
    waits for every copy before this returns, so work queued after it sees the results."""
    dev = torch.device(device)
    cur = torch.cuda.current_stream(dev)
    d_in = [None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev) for t in inputs]
    d_out = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in outputs]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    n = inputs[0].shape[0]
    bounds = [(n * i // groups, n * (i + 1) // groups) for i in range(groups)]
    for lo, hi in bounds:
        if hi == lo:
            continue
        with torch.cuda.stream(s_in):
            for h, d in zip(inputs, d_in):
                if h is not None:
                    d[lo:hi].copy_(h[lo:hi], non_blocking=True)
        cur.wait_stream(s_in)
        run(lo, hi, d_in, d_out)
        s_out.wait_stream(cur)
        with torch.cuda.stream(s_out):
            for h, d in zip(outputs, d_out):
                h[lo:hi].copy_(d[lo:hi], non_blocking=True)
    cur.wait_stream(s_out)


def chunk_fwd_host(q, k, v, g, b, w=None, S0=None, *, mode="gdn2", chunk=64, device="cuda",
                   out=None, groups=None):
    """End-to-end call on host tensors: copies the inputs to the device, runs chunk_fwd and
    copies o and S_T back into host tensors (`out` = (o_host, S_T_host) to reuse pinned
    buffers).  With pinned inputs the (sequence, head) pairs are processed in `groups`
    (default: up to 8) contiguous groups whose copies in both directions overlap the
    computation of the neighbouring groups."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = (torch.empty(B, H, T, dv, dtype=q.dtype, pin_memory=True),
               torch.empty(B, H, dk, dv, dtype=torch.float32, pin_memory=True))
    units = B * H
    ng = min(units, 8) if groups is None else max(1, min(int(groups), units))
    if not q.is_pinned() or ng <= 1:
        to = lambda t: None if t is None else t.to(device, non_blocking=q.is_pinned())
        o_d, S_d = chunk_fwd(to(q), to(k), to(v), to(g), to(b), to(w), to(S0), mode=mode, chunk=chunk)
        out[0].copy_(o_d, non_blocking=True)
        out[1].copy_(S_d, non_blocking=True)
        return out
    flat = lambda t: None if t is None else t.reshape(units, *t.shape[2:])
    ins = [flat(t) for t in (q, k, v, g, b, w, S0)]
    outs = [flat(out[0]), flat(out[1])]

    def run(lo, hi, d, dout):
        one = lambda t: None if t is None else t[lo:hi].unsqueeze(0)
        chunk_fwd(*(one(t) for t in d), mode=mode, chunk=chunk, o=one(dout[0]), S_T=one(dout[1]))
    _pipelined_host_call(ins, outs, ng, run, device)
    return out


def mixer_fwd(q, k, v, xg, xb, xw, z, norm_weight, S0=None, *, mode="gdn2", layout="bhtd",
              b_range=1.0, eps=1e-5, chunk=64, y=None, S_T=None, return_state=True):
    """The recurrence inside its token-mixer block (gdr_mixer_fwd): raw projections in,
    gated output out.  layout "bhtd": q, k, xb [B,H,T,dk], v, xw, z [B,H,T,dv] (scalar
    gates [B,H,T]); "bthd": [B,T,H,d] (scalar gates [B,T,H]).  bf16 except xg (fp32) and
    norm_weight (fp32 [dv]).  Returns (y, S_T) with y in the input layout."""
    if layout not in LAYOUTS:
        raise ValueError(f"unknown layout {layout!r}")
    if layout == "bhtd":
        B, H, T, dk = q.shape
        lead = (B, H, T)
    else:
        B, T, H, dk = q.shape
        lead = (B, T, H)
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    if dt not in DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    gshape, bshape, wshape = _gate_shapes(mode, lead, dk, dv)
    for t, name, shape, tdt in ((q, "q", (*lead, dk), dt), (k, "k", (*lead, dk), dt),
                                (v, "v", (*lead, dv), dt), (xg, "xg", gshape, torch.float32),
                                (xb, "xb", bshape, dt), (z, "z", (*lead, dv), dt),
                                (norm_weight, "norm_weight", (dv,), torch.float32)):
        _check(t, name, shape, tdt, dev)
    if wshape is not None:
        _check(xw, "xw", wshape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if y is None:
        y = torch.empty(*lead, dv, dtype=dt, device=dev)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    rc = gdr_mixer_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(xg), _ptr(xb),
                       _ptr(xw) if wshape is not None else None, _ptr(z), _ptr(norm_weight),
                       _ptr(S0), _ptr(y), _ptr(S_T), B, H, T, dk, dv, chunk, MODES[mode], DTYPES[dt],
                       LAYOUTS[layout], float(b_range), float(eps), _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_mixer_fwd")
    return y, S_T


def mixer_fwd_host(q, k, v, xg, xb, xw, z, norm_weight, S0=None, *, mode="gdn2", layout="bhtd",
                   b_range=1.0, eps=1e-5, device="cuda", out=None, groups=None):
    """mixer_fwd end to end from host tensors; y and S_T come back into host tensors (`out`
    to reuse them).  With pinned inputs the sequences are processed in `groups` (default: up
    to 8) contiguous groups whose copies overlap the computation of the neighbouring
    groups."""
    B = q.shape[0]
    if out is None:
        dv = v.shape[-1]
        H = q.shape[1] if layout == "bhtd" else q.shape[2]
        out = (torch.empty(v.shape[:-1] + (dv,), dtype=q.dtype, pin_memory=True),
               torch.empty(B, H, q.shape[-1], dv, dtype=torch.float32, pin_memory=True))
    ng = min(B, 8) if groups is None else max(1, min(int(groups), B))
    if not q.is_pinned() or ng <= 1:
        to = lambda t: None if t is None else t.to(device, non_blocking=q.is_pinned())
        y_d, S_d = mixer_fwd(to(q), to(k), to(v), to(xg), to(xb), to(xw), to(z), to(norm_weight), to(S0),
                             mode=mode, layout=layout, b_range=b_range, eps=eps)
        out[0].copy_(y_d, non_blocking=True)
        out[1].copy_(S_d, non_blocking=True)
        return out
    nw = norm_weight.to(device, non_blocking=True)

    def run(lo, hi, d, dout):
        sl = lambda t: None if t is None else t[lo:hi]
        q_, k_, v_, xg_, xb_, xw_, z_, S0_ = (sl(t) for t in d)
        mixer_fwd(q_, k_, v_, xg_, xb_, xw_, z_, nw, S0_, mode=mode, layout=layout, b_range=b_range, eps=eps,
                  y=sl(dout[0]), S_T=sl(dout[1]))
    _pipelined_host_call([q, k, v, xg, xb, xw, z, S0], list(out), ng, run, device)
    return out


def chunk_bwd(q, k, v, g, b, w, S0, dO, dS_T=None, *, mode="gdn2", workspace=None, out=None,
              return_dS0=True):
    """Gradients of L = sum(o * dO) + sum(S_T * dS_T) through chunk_fwd (gdr_chunk_bwd).
    Inputs as chunk_fwd; dO like o, dS_T fp32 [B,H,dk,dv] or None.  Returns a dict with dq,
    dk, dv, db, dw (None when the mode has no w) in the input dtype, dg and dS0 in fp32,
    each shaped like its input.  The workspace (uint8 CUDA tensor of at least
    gdr_chunk_bwd_workspace bytes) is allocated here when not given."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    if dt not in DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    gshape, bshape, wshape = _gate_shapes(mode, (B, H, T), dk, dv)
    for t, name, shape, tdt in ((q, "q", (B, H, T, dk), dt), (k, "k", (B, H, T, dk), dt),
                                (v, "v", (B, H, T, dv), dt), (g, "g", gshape, torch.float32),
                                (b, "b", bshape, dt), (dO, "dO", (B, H, T, dv), dt)):
        _check(t, name, shape, tdt, dev)
    if wshape is not None:
        _check(w, "w", wshape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if dS_T is not None:
        _check(dS_T, "dS_T", (B, H, dk, dv), torch.float32, dev)
    need = gdr_chunk_bwd_workspace(B, H, T, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if out is None:
        out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                   dg=torch.empty_like(g), db=torch.empty_like(b),
                   dw=None if wshape is None else torch.empty_like(w),
                   dS0=torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if return_dS0 else None)
    rc = gdr_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w) if wshape is not None else None,
                       _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                       _ptr(out["dg"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]), B, H, T, dk, dv,
                       MODES[mode], DTYPES[dt], _ptr(workspace), workspace.numel() * workspace.element_size(),
                       _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_bwd")
    return out


def decode_step(q, k, v, g, b, w, S, *, mode="gdn2", o=None):
    """One-token step; S [N,H,dk,dv] fp32 is updated in place.  Returns o [N,H,dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    gshape, bshape, wshape = _gate_shapes(mode, (N, H), dk, dv)
    _check(k, "k", (N, H, dk), dt, dev)
    _check(v, "v", (N, H, dv), dt, dev)
    _check(g, "g", gshape, torch.float32, dev)
    _check(b, "b", bshape, dt, dev)
    if wshape is not None:
        _check(w, "w", wshape, dt, dev)
    _check(S, "S", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(N, H, dv, dtype=dt, device=dev)
    rc = gdr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                         _ptr(w) if wshape is not None else None, _ptr(S), _ptr(o),
                         N, H, dk, dv, MODES[mode], DTYPES[dt], _stream())
    if rc != 0:
        raise GdrError(rc, "gdr_decode_step")
    return o
