"""tcgen05 operand layouts and descriptors (tc_util.cuh) against a plain fp32 matmul.

Each case is one operand arrangement the fused chunk kernel relies on: K-major and
MN-major A and B, operands placed inside taller stacked tiles, negated A, and
accumulation onto an existing result."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "tc_probe.cu")
UTIL = os.path.join(os.path.dirname(HERE), "linear_attention_recurrence_wy_b200", "csrc", "tc_util.cuh")
LIB = os.path.join(HERE, "_build", "libtcprobe.so")


def build_probe():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(SRC), os.path.getmtime(UTIL)):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                               "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", tmp, SRC])
        os.replace(tmp, LIB)
    L = ctypes.CDLL(LIB)
    L.tc_probe_gemm.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 11 + [ctypes.c_void_p] * 2
    L.tc_probe_gemm.restype = ctypes.c_int
    return L


CASES = [
    # name,                      N,   K, a_mn, b_mn, neg, reps, a_r0, a_pad, b_r0, b_pad
    ("AP: K/K N64 K128",          64, 128, 0, 0, 0, 1, 0, 0, 0, 0),
    ("WT: A MN in 128-row tile",  64,  64, 1, 0, 0, 1, 0, 64, 0, 0),
    ("UT: A MN",                  64,  64, 1, 0, 0, 1, 0, 0, 0, 0),
    ("ET: -A, B MN, accumulate",  64, 128, 0, 1, 1, 2, 0, 0, 0, 0),
    ("O1: B K-major at row 64",   64, 128, 0, 0, 0, 1, 0, 0, 64, 0),
    ("S: B MN N128 K64",         128,  64, 0, 1, 0, 2, 0, 0, 0, 0),
    ("K/K N128",                 128, 128, 0, 0, 0, 1, 0, 0, 0, 0),
    ("K/K N256 K64",             256,  64, 0, 0, 0, 1, 0, 0, 0, 0),
    ("MN/MN",                     64, 128, 1, 1, 0, 1, 0, 0, 0, 0),
    ("A MN at row 64",            64,  64, 1, 0, 0, 1, 64, 0, 0, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tcgen05_layout(cuda_ok, case):
    L = build_probe()
    name, N, K, a_mn, b_mn, neg, reps, a_r0, a_pad, b_r0, b_pad = case
    M = 128
    g = torch.Generator(device="cuda").manual_seed(N * 7 + K)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.tc_probe_gemm(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, neg, reps,
                         a_r0, a_pad, b_r0, b_pad, st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert st.item() == 0, "bounded wait expired"
    ref = (A.float() @ B.float()) * (-1.0 if neg else 1.0) * reps
    err = (D - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), (name, err)
