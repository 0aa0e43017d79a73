"""Decode step (gdn_decode_step) against the CPU oracle, element by element.

A decode step is Eq. (1) of "論文解説: Qwen3.8-Next の設計" (section "GDNの中身")
applied to one token per sequence; the oracle runs the same token through its
sequential recurrence in fp64.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
import oracle
from parity import TOL, err

pytestmark = pytest.mark.gpu


def _step_inputs(N, H_qk, H_v, dk, dv, dtype, seed, normalize=True):
    x = inputs.draw(N, H_qk, H_v, dk, dv, dtype, seed, "cuda", normalize_qk=normalize)
    S = inputs.draw_state(N, H_v, dk, dv, 0.3, seed + 1, "cuda")
    return x, S


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,H_qk,H_v,dk,dv", [
    (3, 2, 2, 128, 128), (5, 1, 4, 128, 128), (4, 2, 2, 64, 64), (2, 2, 4, 64, 128),
    (3, 3, 3, 128, 64), (1, 1, 1, 128, 128)])
def test_decode_step_matches_oracle(dtype, N, H_qk, H_v, dk, dv):
    x, S = _step_inputs(N, H_qk, H_v, dk, dv, dtype, seed=N * 100 + dk + dv)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, scale=0.8)
    o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref0, scale=0.8)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype]
    assert err(S, S_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_l2norm_flag(dtype):
    x, S = _step_inputs(4, 2, 4, 128, 128, dtype, seed=7, normalize=False)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                              flags=gdn.GDN_FLAG_QK_L2NORM)
    o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref0,
                                      l2norm=True)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype] and err(S, S_ref) < TOL[dtype]


def test_decode_chain_equals_recurrence():
    """Ten chained steps in place equal the oracle's recurrence over ten tokens."""
    N, H, d, steps = 4, 2, 128, 10
    S = inputs.draw_state(N, H, d, d, 0.3, 5, "cuda")
    S0 = S.clone()
    xs, outs = [], []
    for s in range(steps):
        x = inputs.draw(N, H, H, d, d, torch.float32, 50 + s, "cuda")
        xs.append(x)
        outs.append(gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S))
    torch.cuda.synchronize()
    # sequence n = token s of every step
    cat = lambda name: torch.stack([x[name] for x in xs], 1).reshape(N * steps, *xs[0][name].shape[1:])
    cu = np.arange(0, N * steps + 1, steps, dtype=np.int64)
    o_ref, S_ref = oracle.recurrent(cat("q"), cat("k"), cat("v"), cat("g"), cat("beta"), S0=S0,
                                    cu_seqlens=cu)
    o_gpu = torch.stack(outs, 1).reshape(N * steps, H, d)
    assert err(o_gpu, o_ref) < 1e-4 and err(S, S_ref) < 1e-4


def test_decode_full_workload_sampled():
    """The decode workload at full size (256 sequences x 32 heads x 128 steps, bf16 q/k/v,
    fp32 state) in the launch configuration the bench times; 24 sampled (sequence, head)
    pairs are followed through all 128 steps by the oracle, and every output is finite."""
    w = inputs.get(4)
    S = inputs.decode_state(w, "cuda")
    rng = np.random.default_rng(0)
    picks = [(int(n), int(h)) for n, h in zip(rng.integers(0, w.decode_seqs, 24),
                                              rng.integers(0, w.H_v, 24))]
    S0 = torch.stack([S[n, h] for n, h in picks]).cpu()
    keep = {nm: [] for nm in ("q", "k", "v", "g", "beta", "out")}
    for s in range(w.decode_steps):
        x = inputs.decode_step_inputs(w, s, "cuda")
        out = gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
        assert torch.isfinite(out).all()
        for nm in ("q", "k"):
            keep[nm].append(torch.stack([x[nm][n, h // (w.H_v // w.H_qk)] for n, h in picks]).cpu())
        for nm in ("v", "g", "beta"):
            keep[nm].append(torch.stack([x[nm][n, h] for n, h in picks]).cpu())
        keep["out"].append(torch.stack([out[n, h] for n, h in picks]).cpu())
    torch.cuda.synchronize()
    P, T = len(picks), w.decode_steps
    seq = lambda nm: torch.stack(keep[nm], 1).reshape(P * T, 1, -1) if keep[nm][0].dim() > 1 \
        else torch.stack(keep[nm], 1).reshape(P * T, 1)
    cu = np.arange(0, P * T + 1, T, dtype=np.int64)
    o_ref, S_ref = oracle.recurrent(seq("q"), seq("k"), seq("v"), seq("g"), seq("beta"),
                                    S0=S0[:, None], cu_seqlens=cu)
    S_gpu = torch.stack([S[n, h] for n, h in picks]).cpu()
    assert err(seq("out"), o_ref) < TOL[torch.bfloat16]
    assert err(S_gpu, S_ref[:, 0]) < TOL[torch.bfloat16]
