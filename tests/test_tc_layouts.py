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
TRI = os.path.join(os.path.dirname(HERE), "linear_attention_recurrence_wy_b200", "csrc", "tri_inverse.cuh")
LIB = os.path.join(HERE, "_build", "libtcprobe.so")


def build_probe():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(p) for p in (SRC, UTIL, TRI)):
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


def _tri_cases(n=64):
    g = torch.Generator().manual_seed(0)
    low = torch.tril(torch.ones(n, n), -1)
    cases = {
        "small": torch.randn(n, n, generator=g) * 0.1 * low,
        "unit_scale": torch.randn(n, n, generator=g) * (n ** -0.5) * low,
        "all_ones": low.clone(),                                   # inverse is I - subdiagonal
        "pm_half": (torch.rand(n, n, generator=g) - 0.5) * low,
    }
    # the delta-rule structure: A_ij = b_i k_i . k_j exp(gamma_i - gamma_j), keys unit-norm
    k = torch.nn.functional.normalize(torch.randn(n, 128, generator=g), dim=-1)
    b = torch.sigmoid(torch.randn(n, 128, generator=g))
    gam = torch.cumsum(-torch.nn.functional.softplus(torch.randn(n, 128, generator=g)) * 0.1, 0)
    dec = torch.exp((gam[:, None, :] - gam[None, :, :]).clamp(max=0))
    cases["delta_rule"] = torch.einsum("ic,jc,ijc->ij", b * k, k, dec) * low
    return cases


@pytest.mark.parametrize("name", ["small", "unit_scale", "all_ones", "pm_half", "delta_rule"])
def test_triangular_inverse(cuda_ok, name):
    L = build_probe()
    L.tc_probe_tri_inverse.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    L.tc_probe_tri_inverse.restype = ctypes.c_int
    A = _tri_cases()[name]
    Ad = A.float().cuda().contiguous()
    Td = torch.empty_like(Ad)
    assert L.tc_probe_tri_inverse(Ad.data_ptr(), Td.data_ptr(), 1, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    ref = torch.linalg.inv(torch.eye(64, dtype=torch.float64) + A.double())
    T = Td.double().cpu()
    assert torch.all(torch.triu(T, 1) == 0)
    assert torch.all(torch.diagonal(T) == 1)
    err = (T - ref).abs().max().item() / max(1.0, ref.abs().max().item())
    assert err < 2e-3, (name, err)   # TF32 operand rounding (2^-11) in the block products


TS_CASES = [
    # name,                       N,   K, b_mn, neg, reps
    ("E: A=S^T in TMEM, B MN, -A", 64, 128, 1, 1, 2),
    ("O1: B K-major",              64, 128, 0, 0, 1),
    ("O2: K64 B K-major",          64,  64, 0, 0, 2),
    ("S: K64 B MN N128",          128,  64, 1, 0, 1),
]


@pytest.mark.parametrize("case", TS_CASES, ids=[c[0] for c in TS_CASES])
def test_tcgen05_a_from_tmem(cuda_ok, case):
    L = build_probe()
    L.tc_probe_gemm_ts.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 2
    L.tc_probe_gemm_ts.restype = ctypes.c_int
    name, N, K, b_mn, neg, reps = case
    g = torch.Generator(device="cuda").manual_seed(N + K)
    A = torch.randn(128, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((128, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.tc_probe_gemm_ts(A.data_ptr(), B.data_ptr(), D.data_ptr(), N, K, b_mn, neg, reps,
                            st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = (A.float() @ B.float()) * (-1.0 if neg else 1.0) * reps
    err = (D - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), (name, err)
