"""GPU self-checks of the tcgen05 MMA operand layouts and the TMA box load.

These run first (file name order) so that a wrong descriptor or swizzle shows up
as a plain numeric mismatch here before the fused kernels use the same helpers.
Each MMA case is one combination the fused forward uses (M = 128 throughout).
"""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gpu_probe")
SRC = os.path.join(HERE, "tc_probe.cu")
LIB = os.path.join(HERE, "libtcprobe.so")


@pytest.fixture(scope="module")
def probe():
    deps = [SRC] + [os.path.join(HERE, "..", "..", "gated_delta_rule_107_b200", "csrc", f)
                    for f in ("tc_ptx.cuh", "tc_host.cuh", "dr_common.cuh", "tc_inverse.cuh")]
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(p) for p in deps):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                               "-Xcompiler", "-fPIC", "-shared", "-o", LIB, SRC])
    lib = ctypes.CDLL(LIB)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.probe_mma.argtypes = [vp, vp, vp] + [i] * 7
    lib.probe_mma.restype = i
    lib.probe_tma.argtypes = [vp, vp] + [i] * 8
    lib.probe_tma.restype = i
    lib.probe_inverse.argtypes = [vp, vp]
    lib.probe_inverse.restype = i
    return lib


# (name, N, K, a_mn, b_mn): where each is used in the fused forward
CASES = [
    ("P1  [bk;q].k^T     A K-major K=128, B K-major  N=64", 64, 128, 0, 0),
    ("IPT [I;P].T        A K-major K=64,  B MN-major N=64", 64, 64, 0, 1),
    ("P3  R.bK~          A K-major K=64,  B MN-major N=128", 128, 64, 0, 1),
    ("C1  Achain.S       A K-major K=128, B MN-major N=64", 64, 128, 0, 1),
    ("C3  Kbar^T.U       A MN-major K=64, B MN-major N=64", 64, 64, 1, 1),
    ("A MN-major K=128, B K-major N=128", 128, 128, 1, 0),
]


@pytest.mark.parametrize("name,N,K,a_mn,b_mn", CASES, ids=[c[0].split()[0] + f"_N{c[1]}K{c[2]}" for c in CASES])
@pytest.mark.parametrize("neg_a,acc", ((0, 0), (1, 1)))
def test_mma_layout(probe, name, N, K, a_mn, b_mn, neg_a, acc):
    M = 128
    g = torch.Generator().manual_seed(N * 1000 + K + 7 * a_mn + 3 * b_mn)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(K, N, generator=g).to(torch.bfloat16).cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    rc = probe.probe_mma(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, neg_a, acc)
    assert rc == 0, f"probe_mma returned {rc}"
    ref = (A.double() @ B.double()) * (-1.0 if neg_a else 1.0) * (2.0 if acc else 1.0)
    err = (D.double() - ref).abs().max().item()
    assert err <= 1e-3 * max(1.0, ref.abs().max().item()), f"{name}: max err {err}"


@pytest.mark.parametrize("b,h,t0,c0", ((0, 0, 0, 0), (1, 2, 64, 64), (1, 1, 100, 0)))
def test_tma_box_matches_swizzle(probe, b, h, t0, c0):
    Bn, T, H, d = 2, 130, 3, 128
    X = torch.randn(Bn, T, H, d).to(torch.bfloat16).cuda()
    out = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    rc = probe.probe_tma(X.data_ptr(), out.data_ptr(), Bn, T, H, d, b, h, t0, c0)
    assert rc == 0, f"probe_tma returned {rc}"
    ref = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    rows = min(64, T - t0)
    ref[:rows] = X[b, t0:t0 + rows, h, c0:c0 + 64]
    assert torch.equal(out, ref)


@pytest.mark.parametrize("seed,harsh", ((0, False), (1, False), (2, True)))
def test_unit_lower_inverse(probe, seed, harsh):
    """The warpgroup inverse of I + A (diagonal blocks + tf32 column chains) vs fp64."""
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(64, 128, generator=g, dtype=torch.float64)
    if harsh:  # strongly correlated keys, beta = 1: larger entries of A and of its inverse
        k = k + 2.0 * torch.randn(1, 128, generator=g, dtype=torch.float64)
    k = k / k.norm(dim=1, keepdim=True)
    beta = torch.ones(64, dtype=torch.float64) if harsh else torch.sigmoid(torch.randn(64, generator=g,
                                                                                       dtype=torch.float64))
    gcum = torch.cumsum(-torch.nn.functional.softplus(torch.randn(64, generator=g, dtype=torch.float64) - 3), 0)
    A = torch.tril(beta[:, None] * (k @ k.T) * torch.exp(gcum[:, None] - gcum[None, :]), -1)
    ref = torch.linalg.inv(torch.eye(64, dtype=torch.float64) + A)
    Ad = A.float().cuda().contiguous()
    Td = torch.full((64, 64), float("nan"), device="cuda")
    assert probe.probe_inverse(Ad.data_ptr(), Td.data_ptr()) == 0
    Tl = torch.tril(Td.double().cpu())
    err = (Tl - ref).abs().max().item() / ref.abs().max().item()
    assert err < 2e-3, f"inverse rel err {err}"
