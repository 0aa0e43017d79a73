"""Properties of the CUDA path that hold at any size and need no oracle: repeatability,
resumption from a saved state, varlen packing, grouped heads, in-place state, the
agreement of prefill with decode, and of the tensor-core with the CUDA-core kernel.

They follow from Eq. (1) of "論文解説: Qwen3.8-Next の設計" (section "GDNの中身"):
the state after a prefix is all the rule carries forward, sequences never interact,
and a value head only sees its own q/k head."""
from __future__ import annotations

import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
from parity import TOL, err

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _x(lens, H_qk=2, H_v=2, dtype=BF, seed=3, s0=0.05):
    x = inputs.draw(sum(lens), H_qk, H_v, 128, 128, dtype, seed, "cuda")
    x["S0"] = inputs.draw_state(len(lens), H_v, 128, 128, s0, seed + 1, "cuda")
    x["cu"] = inputs.cu_seqlens_of(lens).cuda()
    return x


def _run(x, flags=0, S0="x"):
    S0 = x["S0"] if S0 == "x" else S0
    o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, x["cu"], flags=flags)
    torch.cuda.synchronize()
    return o, S


def test_repeatable_bitwise():
    x = _x([700, 333, 64])
    o1, S1 = _run(x)
    o2, S2 = _run(x)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("T1", [64, 100, 1])
def test_split_run_resumes(T1):
    T = 600
    x = _x([T])
    o, S = _run(x)
    a = {k: (v[:T1] if k in ("q", "k", "v", "g", "beta") else v) for k, v in x.items()}
    a["cu"] = inputs.cu_seqlens_of([T1]).cuda()
    b = {k: (v[T1:] if k in ("q", "k", "v", "g", "beta") else v) for k, v in x.items()}
    b["cu"] = inputs.cu_seqlens_of([T - T1]).cuda()
    oa, Sa = _run(a)
    ob, Sb = _run(b, S0=Sa)
    assert err(torch.cat([oa, ob]), o) < TOL[BF] and err(Sb, S) < TOL[BF]


def test_varlen_packing_equals_separate_calls_bitwise():
    lens = [130, 0, 64, 257]
    x = _x(lens, H_qk=1, H_v=2)
    o, S = _run(x)
    cu = x["cu"].tolist()
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        y = {k: x[k][sl] for k in ("q", "k", "v", "g", "beta")}
        y["S0"] = x["S0"][n:n + 1].contiguous()
        y["cu"] = inputs.cu_seqlens_of([L]).cuda()
        oy, Sy = _run(y)
        assert torch.equal(oy, o[sl]) and torch.equal(Sy[0], S[n])


def test_grouped_heads_equal_repeated_heads_bitwise():
    x = _x([300, 90], H_qk=2, H_v=6)
    o, S = _run(x)
    y = dict(x, q=x["q"].repeat_interleave(3, 1).contiguous(), k=x["k"].repeat_interleave(3, 1).contiguous())
    o2, S2 = _run(y)
    assert torch.equal(o, o2) and torch.equal(S, S2)


def test_in_place_state():
    x = _x([333, 129])
    o, S = _run(x)
    buf = x["S0"].clone()
    o2, S2 = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], buf, x["cu"], S_final=buf)
    torch.cuda.synchronize()
    assert S2.data_ptr() == buf.data_ptr()
    assert torch.equal(o, o2) and torch.equal(S, buf)


@pytest.mark.parametrize("dtype", [torch.float32, BF])
def test_prefill_equals_decode_steps(dtype):
    """prefill over T tokens == T decode steps from the same state (T = 1 and T = 70)."""
    N, T = 3, 70
    x = _x([T] * N, H_qk=1, H_v=2, dtype=dtype)
    o, S = _run(x)
    Sd = x["S0"].clone()
    outs = []
    for t in range(T):
        idx = torch.arange(N, device="cuda") * T + t
        outs.append(gdn.gdn_decode_step(x["q"][idx], x["k"][idx], x["v"][idx], x["g"][idx],
                                        x["beta"][idx], Sd))
        if t == 0:
            assert err(outs[0], o[idx]) < TOL[dtype]
    od = torch.stack(outs, 1).reshape(N * T, 2, 128)
    assert err(od, o) < TOL[dtype] and err(Sd, S) < TOL[dtype]


def test_tensor_core_agrees_with_cuda_core():
    x = _x([1000, 77, 64], H_qk=2, H_v=4)
    o_tc, S_tc = _run(x)
    o_cc, S_cc = _run(x, flags=gdn.GDN_FLAG_FORCE_CUDA_CORE)
    assert err(o_tc, o_cc) < TOL[BF] and err(S_tc, S_cc) < TOL[BF]
