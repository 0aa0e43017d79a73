"""gdn_prefill_static_scratch: the prefill entry point for callers that cannot
allocate device memory (code that runs where cudaMalloc is unavailable or forbidden,
for instance under another runtime's memory pool).  Such a caller passes only its
inputs and outputs; the library supplies the kernel's scratch from a static device
array it keeps itself.  The result must match gdn_prefill (the entry point that
takes a caller-allocated workspace) on the same inputs, within the tolerance the
parity tests use, on two calls in a row (the second call reuses the array the first
one left behind)."""
from __future__ import annotations

import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
from parity import TOL, err

pytestmark = pytest.mark.gpu

CC = gdn.GDN_FLAG_FORCE_CUDA_CORE


def _inputs(lens, dense, dtype, with_s0, seed):
    x = inputs.draw(sum(lens), 2, 4, 128, 128, dtype, seed, "cuda")
    S0 = inputs.draw_state(len(lens), 4, 128, 128, 0.05, seed + 1, "cuda") if with_s0 else None
    if dense:
        B, T = len(lens), lens[0]
        x = {k: t.view(B, T, *t.shape[1:]) for k, t in x.items()}
        cu = None
    else:
        cu = inputs.cu_seqlens_of(lens).cuda()
    return x, S0, cu


@pytest.mark.parametrize("dtype,flags", [(torch.bfloat16, 0), (torch.float32, 0),
                                         (torch.bfloat16, CC)])
@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("with_s0", [True, False])
@pytest.mark.parametrize("want_state", [True, False])
def test_static_scratch_matches_gdn_prefill(dtype, flags, dense, with_s0, want_state):
    lens = [257, 257] if dense else [300, 1, 129, 64, 0]
    x, S0, cu = _inputs(lens, dense, dtype, with_s0, 2024 + 7 * dense + with_s0)
    o_ref, S_ref = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu,
                                   flags=flags)
    torch.cuda.synchronize()
    out = torch.empty_like(x["v"])
    S_final = torch.empty_like(S_ref) if want_state else None
    for _ in range(2):
        out.fill_(float("nan"))
        if S_final is not None:
            S_final.fill_(float("nan"))
        gdn.gdn_prefill_static_scratch(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu,
                                       out=out, S_final=S_final, flags=flags)
        torch.cuda.synchronize()
        assert err(out, o_ref) < TOL[dtype]
        if S_final is not None:
            assert err(S_final, S_ref) < TOL[dtype]


@pytest.mark.parametrize("lens", [[0, 0], []])
def test_static_scratch_empty_batch(lens):
    """No tokens at all (two empty sequences) or no sequences: the early return copies S0
    to S_final (zeros when S0 is None) and launches no kernel that reads the inputs."""
    x, S0, cu = _inputs(lens, False, torch.bfloat16, True, 77)
    N = len(lens)
    out = torch.empty_like(x["v"])
    S_final = torch.full((N, 4, 128, 128), float("nan"), device="cuda")
    gdn.gdn_prefill_static_scratch(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu,
                                   out=out, S_final=S_final)
    torch.cuda.synchronize()
    assert torch.equal(S_final, S0)
    S_final.fill_(float("nan"))
    gdn.gdn_prefill_static_scratch(x["q"], x["k"], x["v"], x["g"], x["beta"], None, cu,
                                   out=out, S_final=S_final)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S_final) == 0
