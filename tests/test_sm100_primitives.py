"""The sm_100a building blocks of the tensor-core prefill, each against a plain
reference: one tcgen05 MMA per operand placement (K-major / MN-major, negated B,
N and K of 64 or 128, A read from TMEM) against torch.matmul in fp32, and one TMA tile load against
the global tensor it copies."""
from __future__ import annotations

import ctypes

import pytest
import torch

import selftest_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return selftest_lib.load()


@pytest.mark.parametrize("variant", [
    0 | 16,            # [K;Q] K^T : A K-major, B K-major, N=64, K=128
    1,                 # K^T T'^T  : A MN-major, B K-major, N=64, K=64
    2 | 4 | 16,        # -S^T W^T  : A K-major, B MN-major (negated), N=64, K=128
    2 | 8,             # U^T K~    : A K-major, B MN-major, N=128, K=64
    0 | 16 | 8,        # A K-major, B K-major, N=128, K=128
    1 | 2 | 16 | 8,    # both MN-major, N=128, K=128
    32 | 64 | 16,      # M=64, N=32, K=128: W S (A K-major, B K-major with 32 rows)
    32 | 64,           # M=64, N=32, K=64:  P U
    32 | 2 | 8,        # M=64, N=128, K=64: T' K with B MN-major
    64 | 1,            # M=128, N=32, K=64: K~^T U with A MN-major
    32 | 64 | 16 | 128,  # M=64, N=32, K=128: W S with S in 64-byte-swizzled rows d
    32 | 64 | 128,       # M=64, N=32, K=64:  P U with U in 64-byte-swizzled rows i
    64 | 1 | 128,        # M=128, N=32, K=64: K~^T U, A MN-major, U in 64-byte rows
    64 | 16 | 128 | 4,   # M=128, N=32, K=128, negated 64-byte-swizzled B
    256 | 16 | 8,        # A from TMEM, B K-major, N=128, K=128: S^T [Q~;W]^T
    256 | 2 | 8,         # A from TMEM, B MN-major, N=128, K=64:  (U dte)^T K
    256,                 # A from TMEM, B K-major, N=64, K=64:    U^T P^T
    256 | 16,            # A from TMEM, B K-major, N=64, K=128
])
def test_umma_placements(L, variant):
    torch.manual_seed(variant)
    M = 64 if variant & 32 else 128
    N = 32 if variant & 64 else (128 if variant & 8 else 64)
    K = 128 if variant & 16 else 64
    A = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda").to(torch.bfloat16)
    D = torch.zeros(M, N, device="cuda", dtype=torch.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.selftest_umma(ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(B.data_ptr()),
                         ctypes.c_void_p(D.data_ptr()), variant, ctypes.c_void_p(st.data_ptr()))
    assert rc == 0 and int(st.item()) == 0
    ref = A.float() @ B.float().T
    if variant & 4:
        ref = -ref
    assert torch.allclose(D, ref, atol=1e-3, rtol=1e-4), (D - ref).abs().max().item()


@pytest.mark.parametrize("t0", [0, 64, 300])
def test_tma_tile_load(L, t0):
    T, H, h = 400, 3, 1
    x = torch.randn(T, H, 128, device="cuda").to(torch.bfloat16)
    out = torch.full((64, 128), -7.0, device="cuda", dtype=torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.selftest_tma(ctypes.c_void_p(x.data_ptr()), T, H, h, t0, ctypes.c_void_p(out.data_ptr()),
                        ctypes.c_void_p(st.data_ptr()))
    assert rc == 0 and int(st.item()) == 0
    rows = min(64, T - t0)
    assert torch.equal(out[:rows], x[t0:t0 + rows, h])
    assert torch.all(out[rows:] == 0)          # past the tensor end: zero fill


def test_cluster_dsmem_copy_and_remote_arrive(L):
    out = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    rc = L.selftest_cluster(ctypes.c_void_p(out.data_ptr()))
    assert rc == 0
    assert out.tolist() == [0] * 8
