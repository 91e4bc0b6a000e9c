"""Host-only tests of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments with the documented status before launching anything.
None of these calls reaches a CUDA API (validation returns first)."""
import ctypes
import os
import re

import pytest

import linear_attention_recurrence_wy_b200 as gdr
from linear_attention_recurrence_wy_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")

OK, NULL, DIM, MODE, DTYPE, ALIGN, WORKSPACE, VALUE = 0, -1, -2, -3, -4, -5, -8, -9


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdr.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdr_chunk_fwd", "gdr_decode_step", "gdr_last_device_error", "gdr_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9):
        s = gdr.gdr_status_string(code)
        assert s.startswith("GDR_")
    assert "unknown" in gdr.gdr_status_string(42)


A = 4096  # a 16-byte aligned fake address: never dereferenced, validation fails first


def call_fwd(q=A, k=A, v=A, g=A, b=A, w=A, S0=None, o=A, ST=None, B=1, H=1, T=8, dk=64, dv=64,
             chunk=64, mode=0, dtype=0):
    return gdr.gdr_chunk_fwd(q, k, v, g, b, w, S0, o, ST, B, H, T, dk, dv, chunk, mode, dtype, None)


def call_dec(q=A, k=A, v=A, g=A, b=A, w=A, S=A, o=A, N=1, H=1, dk=64, dv=64, mode=0, dtype=0):
    return gdr.gdr_decode_step(q, k, v, g, b, w, S, o, N, H, dk, dv, mode, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(mode=5), MODE), (dict(mode=-1), MODE), (dict(dtype=2), DTYPE),
    (dict(dk=48), DIM), (dict(dv=256), DIM), (dict(chunk=128), DIM), (dict(chunk=8), DIM),
    (dict(B=-1), DIM), (dict(T=-1), DIM), (dict(H=-2), DIM),
    (dict(q=None), NULL), (dict(k=None), NULL), (dict(v=None), NULL), (dict(g=None), NULL),
    (dict(b=None), NULL), (dict(o=None), NULL), (dict(w=None), NULL),
    (dict(q=A + 4), ALIGN), (dict(o=A + 2), ALIGN), (dict(S0=A + 8), ALIGN), (dict(ST=A + 12), ALIGN),
    (dict(w=A + 8), ALIGN),
])
def test_chunk_fwd_rejects(L, kw, code):
    assert call_fwd(**kw) == code


def test_chunk_fwd_tied_modes_do_not_need_w(L):
    # w is ignored in KDA/GDN modes; with B = 0 nothing is launched
    assert call_fwd(w=None, mode=1, B=0) == OK
    assert call_fwd(w=None, mode=2, B=0) == OK
    assert call_fwd(w=None, mode=0, B=1) == NULL
    # the b-only and w-only variants carry a w (scalar, resp. per channel)
    assert call_fwd(w=None, mode=3, B=1) == NULL
    assert call_fwd(w=None, mode=4, B=1) == NULL


def test_chunk_fwd_empty_batch_is_a_no_op(L):
    assert call_fwd(q=None, k=None, v=None, g=None, b=None, w=None, o=None, B=0) == OK
    assert call_fwd(q=None, k=None, v=None, g=None, b=None, w=None, o=None, H=0) == OK


@pytest.mark.parametrize("kw,code", [
    (dict(mode=5), MODE), (dict(dtype=-1), DTYPE), (dict(dk=100), DIM), (dict(N=-1), DIM),
    (dict(S=None), NULL), (dict(o=None), NULL), (dict(w=None), NULL), (dict(g=None), NULL),
    (dict(S=A + 4), ALIGN), (dict(q=A + 2), ALIGN),
])
def test_decode_rejects(L, kw, code):
    assert call_dec(**kw) == code


def test_decode_empty_is_a_no_op(L):
    assert call_dec(N=0, S=None, q=None) == OK


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.dirname(gdr.__file__)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                for bad in ("import oracle", "from oracle", "gdr_oracle", "libgdr_oracle"):
                    assert bad not in txt, (f, bad)


def call_split(nseg=4, ws=A, ws_bytes=1 << 30, dk=128, dv=128, chunk=64, dtype=1, T=1024, B=1, H=2):
    return gdr.gdr_chunk_fwd_split(A, A, A, A, A, A, None, A, None, B, H, T, dk, dv, chunk, 0, dtype,
                                   nseg, ws, ws_bytes, None)


def test_split_workspace_size_and_segments(L):
    assert gdr.gdr_chunk_fwd_split_workspace(2, 3, 128, 128, 4) == 3 * 2 * 3 * 4 * 128 * 128 * 4
    assert gdr.gdr_chunk_fwd_split_workspace(1, 1, 100, 128, 4) == 0
    # only the tensor-core shape is split; few sequence-heads and a long sequence do split
    assert gdr.gdr_chunk_fwd_split_segments(1, 16, 16384, 128, 128, 64, 1) > 1
    assert gdr.gdr_chunk_fwd_split_segments(8, 16, 4096, 128, 128, 64, 1) == 1
    assert gdr.gdr_chunk_fwd_split_segments(1, 1, 16384, 64, 64, 64, 1) == 1
    assert gdr.gdr_chunk_fwd_split_segments(1, 1, 16384, 128, 128, 64, 0) == 1


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), WORKSPACE), (dict(ws_bytes=1000), WORKSPACE), (dict(ws=A + 8), WORKSPACE),
    (dict(nseg=0), DIM), (dict(dk=64, nseg=2), DIM), (dict(dtype=0, nseg=2), DIM),
    (dict(chunk=32, nseg=2), DIM),
])
def test_split_rejects(L, kw, code):
    assert call_split(**kw) == code


def call_two_phase(nseg=1, ws=A, ws_bytes=1000, dk=128, dv=128, chunk=64, dtype=1, T=1024, B=1, H=2, mode=0):
    return gdr.gdr_chunk_fwd_two_phase(A, A, A, A, A, A, None, A, None, B, H, T, dk, dv, chunk, mode, dtype,
                                       nseg, ws, ws_bytes, None)


def test_two_phase_workspace_size_and_planner(L):
    rec = 74752                                       # one chunk's record
    # records, then the exact-path list (a count and one index per chunk, 16-byte padded),
    # then the sequence split's three state arrays when the state pass is split
    assert gdr.gdr_chunk_fwd_two_phase_workspace(2, 3, 1000, 128, 128, 64, 1) == 6 * 16 * rec + 400
    assert gdr.gdr_chunk_fwd_two_phase_workspace(2, 3, 1000, 128, 128, 64, 4) == \
        6 * 16 * rec + 400 + 3 * 6 * 4 * 128 * 128 * 4
    assert gdr.gdr_chunk_fwd_two_phase_workspace(1, 1, 100, 64, 64, 64, 1) == 0
    assert gdr.gdr_chunk_fwd_two_phase_workspace(1, 1, 100, 128, 128, 32, 1) == 0
    assert gdr.gdr_chunk_fwd_two_phase_workspace(1, 1, 100, 128, 128, 64, 0) == 0
    # the planner (this host has no GPU: 148 SMs assumed), with its measured constants, takes
    # the two-phase path for few sequence-heads (64 at T = 2K, one state pass; 16 at T = 16K,
    # a split state pass), and the fused kernel when the sequence-heads fill the GPU (128 at
    # T = 4K) or the sequences are short (256 at T = 1K)
    assert gdr.gdr_chunk_fwd_two_phase_segments(4, 16, 2048, 128, 128, 64, 1) == 1
    assert gdr.gdr_chunk_fwd_two_phase_segments(1, 16, 16384, 128, 128, 64, 1) > 1
    assert gdr.gdr_chunk_fwd_two_phase_segments(8, 16, 4096, 128, 128, 64, 1) == 0
    assert gdr.gdr_chunk_fwd_two_phase_segments(16, 16, 1024, 128, 128, 64, 1) == 0
    assert gdr.gdr_chunk_fwd_two_phase_segments(1, 16, 16384, 64, 64, 64, 1) == 0
    assert gdr.gdr_chunk_fwd_two_phase_segments(1, 16, 16384, 128, 128, 64, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), WORKSPACE), (dict(ws_bytes=1 << 20), WORKSPACE), (dict(ws=A + 8), WORKSPACE),
    (dict(nseg=0), DIM), (dict(dk=64), DIM), (dict(dtype=0), DIM), (dict(chunk=32), DIM), (dict(mode=6), MODE),
    (dict(T=-1), DIM),
])
def test_two_phase_rejects(L, kw, code):
    assert call_two_phase(**kw) == code


def test_two_phase_empty_is_a_no_op(L):
    assert call_two_phase(B=0) == OK
    assert call_two_phase(H=0) == OK


def call_mixer(q=A, k=A, v=A, xg=A, xb=A, xw=A, z=A, nw=A, S0=None, y=A, ST=None, B=1, H=2, T=8,
               dk=128, dv=128, chunk=64, mode=0, dtype=1, layout=1, b_range=1.0, eps=1e-5):
    return gdr.gdr_mixer_fwd(q, k, v, xg, xb, xw, z, nw, S0, y, ST, B, H, T, dk, dv, chunk, mode, dtype,
                             layout, b_range, eps, None)


@pytest.mark.parametrize("kw,code", [
    (dict(mode=7), MODE), (dict(dtype=0), DTYPE), (dict(dtype=3), DTYPE), (dict(dk=64), DIM),
    (dict(dv=64), DIM), (dict(chunk=32), DIM), (dict(T=-1), DIM), (dict(layout=2), VALUE),
    (dict(layout=-1), VALUE), (dict(eps=0.0), VALUE), (dict(eps=-1.0), VALUE),
    (dict(eps=float("nan")), VALUE), (dict(eps=float("inf")), VALUE), (dict(b_range=-0.5), VALUE),
    (dict(b_range=float("nan")), VALUE), (dict(q=None), NULL), (dict(xg=None), NULL),
    (dict(xb=None), NULL), (dict(xw=None), NULL), (dict(z=None), NULL), (dict(nw=None), NULL),
    (dict(y=None), NULL), (dict(z=A + 2), ALIGN), (dict(nw=A + 4), ALIGN), (dict(xg=A + 8), ALIGN),
])
def test_mixer_rejects(L, kw, code):
    assert call_mixer(**kw) == code


def test_mixer_tied_modes_and_empty_batch(L):
    # xw is ignored in the tied modes; with B = 0 nothing is launched
    assert call_mixer(xw=None, mode=1, B=0) == OK
    assert call_mixer(xw=None, mode=2, B=0) == OK
    assert call_mixer(q=None, k=None, v=None, xg=None, xb=None, xw=None, z=None, nw=None, y=None, B=0) == OK


def call_bwd(q=A, k=A, v=A, g=A, b=A, w=A, S0=None, dO=A, dST=None, dq=A, dk_=A, dv_=A, dg=A, db=A, dw=A,
             dS0=A, B=1, H=2, T=40, dk=64, dv=64, mode=0, dtype=0, ws=A, ws_bytes=1 << 40):
    return gdr.gdr_chunk_bwd(q, k, v, g, b, w, S0, dO, dST, dq, dk_, dv_, dg, db, dw, dS0, B, H, T, dk, dv, mode,
                             dtype, ws, ws_bytes, None)


def test_bwd_workspace_size(L):
    # two fp32 states per 32-token chunk and sequence-head, then a count and one index per
    # 64-token span (the spans the tensor-core kernel leaves to the CUDA-core one), padded
    # to 16 bytes
    states = 2 * 2 * 3 * 4 * 64 * 32 * 4
    assert gdr.gdr_chunk_bwd_workspace(2, 3, 100, 64, 32) == states + 64   # (1 + 2*3*2) ints
    assert gdr.gdr_chunk_bwd_workspace(1, 1, 64, 128, 128) == 2 * 2 * 128 * 128 * 4 + 16
    assert gdr.gdr_chunk_bwd_workspace(2, 3, 0, 64, 32) == 0
    assert gdr.gdr_chunk_bwd_workspace(2, 3, 10, 48, 32) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(mode=9), MODE), (dict(dtype=5), DTYPE), (dict(dk=24), DIM), (dict(T=-1), DIM), (dict(B=-1), DIM),
    (dict(q=None), NULL), (dict(dO=None), NULL), (dict(dq=None), NULL), (dict(dg=None), NULL),
    (dict(db=None), NULL), (dict(dw=None), NULL), (dict(w=None), NULL),
    (dict(ws=None), WORKSPACE), (dict(ws_bytes=100), WORKSPACE),
    (dict(dq=A + 2), ALIGN), (dict(ws=A + 8), ALIGN), (dict(dS0=A + 4), ALIGN),
])
def test_bwd_rejects(L, kw, code):
    assert call_bwd(**kw) == code


def test_bwd_tied_modes_need_no_w(L):
    assert call_bwd(w=None, dw=None, mode=1, B=0) == OK
    assert call_bwd(q=None, k=None, v=None, g=None, b=None, w=None, dO=None, dq=None, dk_=None, dv_=None,
                    dg=None, db=None, dw=None, dS0=None, H=0) == OK
