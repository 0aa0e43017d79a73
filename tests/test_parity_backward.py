"""Backward pass (gdn_backward) against the CPU oracle's reverse-mode differentiation of
Eq. (1) ("論文解説: Qwen3.8-Next の設計", section "GDNの中身"), element by element.

The kernel computes in fp32 from the same (bf16-rounded) inputs the oracle reads in fp64,
so both input types are held to the fp32 tolerance, max|x - ref| / max|ref| <= 1e-4, on
every gradient separately.  The oracle itself is pinned by finite differences of the
forward oracle (tests/test_oracle.py).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
import oracle
from oracle.backward import backward as oracle_backward
from parity import err

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _case(lens, H_qk, H_v, dk, dv, dtype, seed, s0_std=0.05, with_dSf=True):
    w = inputs.small("bw", lens, H_qk, H_v, dk, dv, dtype, s0_std=s0_std)
    x = inputs.prefill_inputs(w, device="cuda", seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    d_out = torch.randn(x["v"].shape, generator=gen).to(dtype).cuda()
    dSf = (torch.randn(len(lens), H_v, dk, dv, generator=gen) * 0.1).cuda() if with_dSf else None
    return x, d_out, dSf


def _check(x, d_out, dSf, scale=1.0, flags=0, g=None, beta=None):
    grads = gdn.gdn_backward(x["q"], x["k"], x["v"], x["g"] if g is None else g,
                             x["beta"] if beta is None else beta, d_out, x["S0"], dSf,
                             x["cu_seqlens"], scale=scale, flags=flags)
    torch.cuda.synchronize()
    gg, bb = (x["g"], x["beta"]) if g is None else oracle.gates_from_logits(g, beta)
    ref = oracle_backward(x["q"], x["k"], x["v"], gg, bb, x["S0"], d_out, dSf,
                          x["cu_seqlens"].cpu().numpy(), scale=scale)
    names = ["dq", "dk", "dv", "dg", "dbeta", "dS0"]
    ref = dict(zip(names, ref))
    if g is not None:
        # chain rule through the gate prologue: g = -softplus(a), beta = sigmoid(b)
        a = g.double().cpu().numpy(); b = beta.double().cpu().numpy()
        ref["dg"] = ref["dg"] * (-1.0 / (1.0 + np.exp(-a)))
        sb = 1.0 / (1.0 + np.exp(-b))
        ref["dbeta"] = ref["dbeta"] * sb * (1.0 - sb)
    for n in names:
        e = err(grads[n], ref[n])
        assert e < TOL, (n, e)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("lens,H_qk,H_v,dk,dv", [
    ([130, 1, 64, 200], 2, 4, 128, 128),       # ragged, GVA, one token, chunk-exact
    ([150], 1, 1, 64, 64),
    ([70, 129], 2, 2, 128, 64),
    ([65, 3], 1, 2, 64, 128),
    ([70, 0, 5, 1], 2, 2, 128, 128),          # an empty sequence passes dS_final to dS0
])
def test_backward_matches_oracle(dtype, lens, H_qk, H_v, dk, dv):
    x, d_out, dSf = _case(lens, H_qk, H_v, dk, dv, dtype, seed=sum(lens) + dk + dv)
    _check(x, d_out, dSf, scale=0.8)


def test_backward_without_state_gradients():
    """No S0 and no dS_final: the loss reaches the state only through the outputs."""
    x, d_out, _ = _case([100, 37], 2, 2, 128, 128, torch.bfloat16, seed=5, s0_std=0.0,
                        with_dSf=False)
    _check(x, d_out, None)


def test_backward_gate_logits():
    """With GDN_FLAG_GATE_LOGITS, dg and dbeta are the gradients with respect to the logits."""
    x, d_out, dSf = _case([90, 40], 1, 2, 128, 128, torch.float32, seed=9)
    gen = torch.Generator().manual_seed(10)
    a = (torch.randn(x["g"].shape, generator=gen) * 2).cuda()
    b = (torch.randn(x["beta"].shape, generator=gen) * 2).cuda()
    _check(x, d_out, dSf, flags=gdn.GDN_FLAG_GATE_LOGITS, g=a, beta=b)


def test_backward_dense_batch_layout():
    """The dense [B, T] form gives the same gradients as its varlen packing."""
    B, T, H, d = 2, 96, 2, 128
    x, d_out, dSf = _case([T] * B, H, H, d, d, torch.bfloat16, seed=21)
    view = lambda t: t.view(B, T, *t.shape[1:])
    dense = gdn.gdn_backward(view(x["q"]), view(x["k"]), view(x["v"]), view(x["g"]),
                             view(x["beta"]), view(d_out), x["S0"], dSf)
    packed = gdn.gdn_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_out, x["S0"], dSf,
                              x["cu_seqlens"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert err(dense[n].reshape(packed[n].shape), packed[n].double().cpu()) < 1e-6, n


def test_backward_is_repeatable_up_to_atomics():
    """Two calls agree to rounding: dv and dS0 bit for bit (each element has one writer),
    the atomically accumulated dq, dk, dg, dbeta within float rounding."""
    x, d_out, dSf = _case([150, 40], 2, 4, 128, 128, torch.bfloat16, seed=31)
    a = gdn.gdn_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_out, x["S0"], dSf,
                         x["cu_seqlens"])
    b = gdn.gdn_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_out, x["S0"], dSf,
                         x["cu_seqlens"])
    torch.cuda.synchronize()
    assert torch.equal(a["dv"], b["dv"]) and torch.equal(a["dS0"], b["dS0"])
    for n in ("dq", "dk", "dg", "dbeta"):
        assert err(a[n], b[n].double().cpu()) < 1e-5, n
