"""Gate prologue (GDN_FLAG_GATE_LOGITS) against the CPU oracle.

The decay gate alpha = exp(g) and the write strength beta must lie in (0, 1) ("論文解説:
Qwen3.8-Next の設計", section "GDNの中身", the text under Eq. (1)).  With the flag, the
g and beta arrays carry unconstrained logits a, b and every kernel forms
g = -softplus(a), beta = sigmoid(b) as it loads them; the oracle applies the same map in
fp64 (oracle.gates_from_logits) and then runs its sequential recurrence.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
import oracle
from parity import TOL, err, oracle_prefill

pytestmark = pytest.mark.gpu

GL = gdn.GDN_FLAG_GATE_LOGITS


def _logits(shape, seed, device="cuda"):
    gen = torch.Generator().manual_seed(seed)
    a = torch.randn(shape, generator=gen, dtype=torch.float32) * 2.0
    b = torch.randn(shape, generator=gen, dtype=torch.float32) * 2.0
    return a.to(device), b.to(device)


def _with_gates(x, a, b):
    g, beta = oracle.gates_from_logits(a, b)
    y = dict(x)
    y["g"] = torch.from_numpy(g)
    y["beta"] = torch.from_numpy(beta)
    return y


@pytest.mark.parametrize("dtype,flags", [(torch.bfloat16, 0), (torch.float32, 0),
                                         (torch.bfloat16, gdn.GDN_FLAG_FORCE_CUDA_CORE)])
def test_prefill_gate_logits(dtype, flags):
    lens = [130, 64, 1, 257]
    x = inputs.prefill_inputs(inputs.small("gate", lens, 2, 4, 128, 128, dtype, s0_std=0.05),
                              device="cuda")
    a, b = _logits(x["g"].shape, 11)
    o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], a, b, x["S0"], x["cu_seqlens"],
                           flags=flags | GL)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(_with_gates(x, a.cpu(), b.cpu()))
    assert err(o, o_ref) < TOL[dtype]
    assert err(S, S_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_step_gate_logits(dtype):
    N, H, d = 5, 4, 128
    x = inputs.draw(N, 2, H, d, d, dtype, 21, "cuda")
    S = inputs.draw_state(N, H, d, d, 0.3, 22, "cuda")
    a, b = _logits((N, H), 23)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_step(x["q"], x["k"], x["v"], a, b, S, flags=GL)
    g, beta = oracle.gates_from_logits(a.cpu(), b.cpu())
    o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], g, beta, S_ref0)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype] and err(S, S_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_multi_gate_logits(dtype):
    N, T, H, d = 4, 3, 4, 128
    x = inputs.draw(N * T, 2, H, d, d, dtype, 31, "cuda")
    x = {key: t.reshape((N, T) + tuple(t.shape[1:])).contiguous() for key, t in x.items()}
    S = inputs.draw_state(N, H, d, d, 0.3, 32, "cuda")
    a, b = _logits((N, T, H), 33)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], a, b, S, flags=GL)
    g, beta = oracle.gates_from_logits(a.cpu(), b.cpu())
    o_ref, S_ref = oracle.decode_multi(x["q"], x["k"], x["v"], g, beta, S_ref0)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype] and err(S, S_ref) < TOL[dtype]


def test_gate_logits_extremes_stay_finite():
    """Logits of +-60 (alpha and beta at the ends of (0, 1)) give finite results that
    match the oracle."""
    lens = [100]
    x = inputs.prefill_inputs(inputs.small("gx", lens, 1, 2, 128, 128, torch.float32),
                              device="cuda")
    a, b = _logits(x["g"].shape, 41)
    a = torch.where(a > 0, torch.full_like(a, 60.0), torch.full_like(a, -60.0))
    b = torch.where(b > 0, torch.full_like(b, 60.0), torch.full_like(b, -60.0))
    o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], a, b, None, x["cu_seqlens"], flags=GL)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    o_ref, S_ref = oracle_prefill(_with_gates(x, a.cpu(), b.cpu()))
    assert err(o, o_ref) < TOL[torch.float32] and err(S, S_ref) < TOL[torch.float32]
