"""Multi-token decode / draft verification (gdn_decode_multi) against the CPU oracle.

T consecutive tokens per (sequence, value head) in one call are Eq. (1) of "論文解説:
Qwen3.8-Next の設計" (section "GDNの中身") applied T times in order; the oracle runs
the same tokens through its sequential recurrence in fp64, and the committed state is
the recurrence's state after the accepted prefix.
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


def _multi_inputs(N, T, H_qk, H_v, dk, dv, dtype, seed, normalize=True):
    x = inputs.draw(N * T, H_qk, H_v, dk, dv, dtype, seed, "cuda", normalize_qk=normalize)
    x = {key: t.reshape((N, T) + tuple(t.shape[1:])).contiguous() for key, t in x.items()}
    S = inputs.draw_state(N, H_v, dk, dv, 0.3, seed + 1, "cuda")
    return x, S


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,T,H_qk,H_v,dk,dv", [
    (3, 1, 2, 2, 128, 128), (4, 2, 1, 4, 128, 128), (3, 5, 2, 2, 64, 64), (2, 8, 2, 4, 64, 128),
    (5, 3, 3, 3, 128, 64), (1, 8, 1, 1, 128, 128)])
def test_decode_multi_matches_oracle(dtype, N, T, H_qk, H_v, dk, dv):
    x, S = _multi_inputs(N, T, H_qk, H_v, dk, dv, dtype, seed=N * 100 + T * 10 + dk + dv)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S, scale=0.8)
    o_ref, S_ref = oracle.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref0, scale=0.8)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype]
    assert err(S, S_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_multi_commits_a_prefix(dtype):
    """Outputs cover all T tokens; each sequence keeps the state after its own accepted
    prefix (0 = unchanged, T = all), as a draft verifier needs."""
    N, T = 6, 5
    x, S = _multi_inputs(N, T, 2, 4, 128, 128, dtype, seed=77)
    commit = torch.tensor([0, 1, 2, 5, 3, 7], dtype=torch.int32, device="cuda")  # 7 clamps to T
    S_ref0 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S, n_commit=commit)
    o_ref, S_ref = oracle.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref0,
                                       n_commit=commit.cpu().numpy())
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[dtype]
    assert err(S, S_ref) < TOL[dtype]
    assert torch.equal(S[0], S_ref0[0])          # nothing committed: untouched bit for bit


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_multi_equals_chained_single_steps(dtype):
    """Per token the arithmetic is the single step's, in the same order: T tokens in one
    call reproduce T calls of gdn_decode_step exactly."""
    N, T = 5, 6
    x, S = _multi_inputs(N, T, 2, 4, 128, 128, dtype, seed=91)
    S1 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
    outs = [gdn.gdn_decode_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                                x["v"][:, t].contiguous(), x["g"][:, t].contiguous(),
                                x["beta"][:, t].contiguous(), S1) for t in range(T)]
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(outs, dim=1))
    assert torch.equal(S, S1)


def test_decode_multi_l2norm_flag():
    x, S = _multi_inputs(3, 4, 2, 4, 128, 128, torch.bfloat16, seed=13, normalize=False)
    S_ref0 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                               flags=gdn.GDN_FLAG_QK_L2NORM)
    o_ref, S_ref = oracle.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref0,
                                       l2norm=True)
    torch.cuda.synchronize()
    assert err(out, o_ref) < TOL[torch.bfloat16] and err(S, S_ref) < TOL[torch.bfloat16]


def test_decode_multi_full_size_sampled():
    """The bench's verification workload (256 sequences x 32 heads, d = 128, T = 4 tokens,
    fp32 state ~ N(0, 0.02)), checked on sampled (sequence, head) pairs."""
    N, T, H, d = 256, 4, 32, 128
    x, _ = _multi_inputs(N, T, H, H, d, d, torch.bfloat16, seed=4040)
    S = inputs.draw_state(N, H, d, d, 0.02, 4041, "cuda")
    commit = torch.randint(0, T + 1, (N,), generator=torch.Generator().manual_seed(4042),
                           dtype=torch.int32).cuda()
    S_ref0 = S.clone()
    out = gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S, n_commit=commit)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4043)
    seqs = sorted(set(rng.integers(0, N, 6).tolist()))
    for n in seqs:
        sl = slice(n, n + 1)
        o_ref, S_ref = oracle.decode_multi(x["q"][sl], x["k"][sl], x["v"][sl], x["g"][sl],
                                           x["beta"][sl], S_ref0[sl],
                                           n_commit=commit[sl].cpu().numpy())
        assert err(out[sl], o_ref) < TOL[torch.bfloat16]
        assert err(S[sl], S_ref) < TOL[torch.bfloat16]
