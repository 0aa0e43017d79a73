"""The B200 costs the tensor-core prefill's design rests on, measured by the probes in
tests/csrc/umma_selftest.cu (one GPU; cycles from clock64).  The assertions are loose
sanity bounds; the printed figures (pytest -s) are the ones the design cites:
tcgen05.mma issue and completion, try_wait on a completed barrier, remote mbarrier
arrives (release vs relaxed), DSMEM bulk copies from one SM, bulk stores to and bulk
loads from global memory."""
from __future__ import annotations

import ctypes

import pytest
import torch

import selftest_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return selftest_lib.load()


def _median(t):
    v = sorted(t.tolist())
    return v[len(v) // 2]


def test_mma_issue_and_wait_costs(L):
    reps = 40
    cyc = torch.zeros(3 * reps, dtype=torch.int64, device="cuda")
    assert L.selftest_contention(0, reps, 60000, ctypes.c_void_p(cyc.data_ptr())) == 0
    c = cyc.view(reps, 3).cpu()[8:]
    issue, total, wait = _median(c[:, 0]), _median(c[:, 1]), _median(c[:, 2])
    print(f"8 x tcgen05.mma (M64 N32 K16): issue {issue} cycles, issue+complete {total}; "
          f"try_wait on a completed phase {wait}")
    assert 8 <= issue < 20000 and issue < total < 40000 and 0 < wait < 2000


def test_remote_arrive_and_bulk_copy_costs(L):
    reps = 12
    g = torch.zeros(131072 + reps * 65536, dtype=torch.uint8, device="cuda")
    cyc = torch.zeros(6 * reps, dtype=torch.int64, device="cuda")
    assert L.selftest_movement(ctypes.c_void_p(g.data_ptr()), 40960, reps, ctypes.c_void_p(cyc.data_ptr())) == 0
    c = cyc.view(reps, 6).cpu()[4:]
    m = [_median(c[:, i]) for i in range(6)]
    print(f"40 KB bulk store: read {m[0]}, complete {m[1]}; 40 KB bulk load from L2 {m[2]}; "
          f"4 remote arrives release {m[3]}, relaxed {m[4]}; cold 40 KB load {m[5]}")
    assert all(0 < x < 10**6 for x in m)
    assert m[4] < m[3]                       # relaxed arrives are the cheap ones


def test_dsmem_bulk_copy_rate(L):
    reps = 12
    cyc = torch.zeros(reps, dtype=torch.int64, device="cuda")
    assert L.selftest_dsmem_bw(28 * 1024, 15, reps, ctypes.c_void_p(cyc.data_ptr())) == 0
    med = _median(cyc.cpu()[4:])
    print(f"4 x 28 KB DSMEM bulk copies from one SM: {med} cycles = {4 * 28 * 1024 / med:.1f} B/cycle")
    assert 0 < med < 10**6
