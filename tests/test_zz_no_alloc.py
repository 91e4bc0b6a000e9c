"""gdr_chunk_fwd_split_noalloc: the sequence split for callers that cannot allocate
device memory (plugins whose host framework owns every device allocation, latency-
critical loops that cannot afford a cudaMalloc).  Its workspace is a fixed array inside
the library.  This file is collected last on purpose: a failure here leaves every other
test already run.  Each check calls the new entry point through the C ABI twice in a
row and compares with the caller-workspace entry point, gdr_chunk_fwd_split."""
import pytest
import torch

import workload
from util import assert_close, np64, to_dev

gdr = pytest.importorskip("linear_attention_recurrence_wy_b200")
pytestmark = pytest.mark.gpu

WORKSPACE = -8


def _ptrs(d):
    p = lambda t: None if t is None else t.data_ptr()
    return [p(d[x]) for x in ("q", "k", "v", "g", "b")] + [p(d["w"]) if d["mode"] == "gdn2" else None]


@pytest.mark.parametrize("mode,nseg", [("gdn2", 4), ("kda", 3)])
def test_noalloc_matches_workspace_entry_twice(cuda_ok, mode, nseg):
    B, H, T = 1, 4, 2000
    d = to_dev(workload.make_small(B, H, T, 128, 128, mode=mode, dtype="bf16", seed=11 + nseg,
                                   g_scale=0.1, s0_std=0.05))
    o_ref, S_ref = gdr.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                       mode=mode, nseg=nseg)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = gdr.gdr_chunk_fwd_split_noalloc(*_ptrs(d), d["S0"].data_ptr(), o.data_ptr(),
                                             S.data_ptr(), B, H, T, 128, 128, 64,
                                             gdr.MODES[mode], 1, nseg, stream)
        assert rc == 0, gdr.gdr_status_string(rc)
        torch.cuda.synchronize()
        assert gdr.gdr_last_device_error(stream) == 0
        assert_close("o", np64(o), np64(o_ref), "bf16")
        assert_close("S_T", np64(S), np64(S_ref), "bf16")


def _call(d, o, S, B, H, T, nseg, mode="gdn2"):
    return gdr.gdr_chunk_fwd_split_noalloc(*_ptrs(d), None if d["S0"] is None else d["S0"].data_ptr(),
                                           o.data_ptr(), None if S is None else S.data_ptr(),
                                           B, H, T, 128, 128, 64, gdr.MODES[mode], 1, nseg,
                                           torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    # 2 x 64 sequence-heads in 8 segments need 48 MiB of workspace (> 24 MiB built in):
    # rejected before anything is launched, so the output keeps its NaNs
    B, H, T = 2, 64, 1024
    assert gdr.gdr_chunk_fwd_split_workspace(B, H, 128, 128, 8) > 24 << 20
    x = torch.zeros(B, H, T, 128, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(B, H, T, 128, device="cuda")
    o = torch.full_like(x, float("nan"))
    rc = gdr.gdr_chunk_fwd_split_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(), g.data_ptr(),
                                         x.data_ptr(), x.data_ptr(), None, o.data_ptr(), None,
                                         B, H, T, 128, 128, 64, 0, 1, 8,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(o.float()).all()


def test_noalloc_request_exactly_at_its_limit(cuda_ok):
    # 32 sequence-heads x 4 segments at d = 128: 3 x 128 x 64 KiB = 24 MiB, the whole array
    B, H, T, nseg = 1, 32, 1024, 4
    assert gdr.gdr_chunk_fwd_split_workspace(B, H, 128, 128, nseg) == 24 << 20
    d = to_dev(workload.make_small(B, H, T, 128, 128, mode="gdn2", dtype="bf16", seed=5,
                                   g_scale=0.1, s0_std=0.05))
    o_ref, S_ref = gdr.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                       mode="gdn2", nseg=nseg)
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = _call(d, o, S, B, H, T, nseg)
        assert rc == 0, gdr.gdr_status_string(rc)
        torch.cuda.synchronize()
        assert gdr.gdr_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
        assert_close("o", np64(o), np64(o_ref), "bf16")
        assert_close("S_T", np64(S), np64(S_ref), "bf16")


def test_noalloc_reports_argument_errors_and_runs_one_segment_unsplit(cuda_ok):
    B, H, T = 1, 2, 200
    d = to_dev(workload.make_small(B, H, T, 128, 128, mode="gdn2", dtype="bf16", seed=6,
                                   g_scale=0.1, s0_std=0.05))
    o = torch.empty_like(d["v"])
    S = torch.empty_like(d["S0"])
    # a NULL input: the split's own status, not a scratch-lookup failure
    rc = gdr.gdr_chunk_fwd_split_noalloc(None, *_ptrs(d)[1:], d["S0"].data_ptr(), o.data_ptr(),
                                         S.data_ptr(), B, H, T, 128, 128, 64, 0, 1, 2,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == gdr.gdr_chunk_fwd_split(None, *_ptrs(d)[1:], d["S0"].data_ptr(), o.data_ptr(),
                                         S.data_ptr(), B, H, T, 128, 128, 64, 0, 1, 2, None, 0,
                                         torch.cuda.current_stream().cuda_stream) != 0
    # one segment: the unsplit forward, equal to gdr_chunk_fwd
    o1, S1 = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode="gdn2")
    assert _call(d, o, S, B, H, T, 1) == 0
    torch.cuda.synchronize()
    assert torch.equal(o, o1) and torch.equal(S, S1)
