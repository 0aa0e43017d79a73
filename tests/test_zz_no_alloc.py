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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_gdn_prefill(dtype):
    lens = [300, 1, 129, 64]
    x = inputs.draw(sum(lens), 2, 4, 128, 128, dtype, 2024, "cuda")
    S0 = inputs.draw_state(len(lens), 4, 128, 128, 0.05, 2025, "cuda")
    cu = inputs.cu_seqlens_of(lens).cuda()
    o_ref, S_ref = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu)
    torch.cuda.synchronize()
    out = torch.empty_like(x["v"])
    S_final = torch.empty_like(S_ref)
    for _ in range(2):
        out.fill_(float("nan"))
        S_final.fill_(float("nan"))
        gdn.gdn_prefill_static_scratch(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu,
                                       out=out, S_final=S_final)
        torch.cuda.synchronize()
        assert err(out, o_ref) < TOL[dtype]
        assert err(S_final, S_ref) < TOL[dtype]
