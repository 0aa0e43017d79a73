"""The C ABI's calls inside CUDA graphs: captured once, replayed, bit-identical to eager.

Serving loops replay a decode step as a CUDA graph rather than relaunching each kernel.
Every entry point enqueues only kernels on the caller's stream (no allocation, no host
synchronisation), so it must capture.  Each replay must also give the eager call's result
bit for bit, including the QSA indexer, whose workspace must come back zeroed for the next
replay.
"""
from __future__ import annotations

import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                      # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_steps_replay():
    """Four decode steps (state updated in place) as one graph."""
    w = inputs.get(4)
    N, H = 16, 8
    S_init = inputs.draw_state(N, H, 128, 128, 0.02, 71, DEV)
    xs = [inputs.draw(N, H, H, 128, 128, torch.bfloat16, 72 + s, DEV) for s in range(4)]
    outs = [torch.empty_like(x["v"]) for x in xs]
    S = S_init.clone()

    def steps():
        for x, o in zip(xs, outs):
            gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out=o)

    S.copy_(S_init)
    steps()
    torch.cuda.synchronize()
    want_S, want_o = S.clone(), [o.clone() for o in outs]
    S.copy_(S_init)
    g = _capture(steps)
    for _ in range(2):
        S.copy_(S_init)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(S, want_S)
        for o, wo in zip(outs, want_o):
            assert torch.equal(o, wo)
    assert w.decode_steps > 0


@pytest.mark.parametrize("schedule", [0, -1, 128, -2])
def test_prefill_replay(schedule):
    """Every prefill schedule captures: automatic, one unit per sequence, 128-token segments
    (unit table, local and transfer chains, scan, correction) and the cluster kernel."""
    lens = [300, 517]
    x = inputs.draw(sum(lens), 4, 8, 128, 128, torch.bfloat16, 73, DEV)
    S0 = inputs.draw_state(2, 8, 128, 128, 0.05, 74, DEV)
    cu = inputs.cu_seqlens_of(lens).to(DEV)
    out = torch.empty_like(x["v"])
    Sf = torch.empty(2, 8, 128, 128, device=DEV)
    gdn.gdn_set_prefill_segment_tokens(schedule)
    try:
        ws = gdn.prefill_workspace(2, sum(lens), 8, 128, 128)
        call = lambda: gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, cu,
                                       out=out, S_final=Sf, workspace=ws)
        call()
        torch.cuda.synchronize()
        want_o, want_S = out.clone(), Sf.clone()
        g = _capture(call)
        for _ in range(2):
            out.zero_(); Sf.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, want_o) and torch.equal(Sf, want_S)
    finally:
        gdn.gdn_set_prefill_segment_tokens(0)
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK


def test_qsa_compress_and_index_replay():
    lens = [40_000, 9_001, 2]
    k = inputs.qsa_keys(sum(lens), 75, DEV)
    cu = inputs.qsa_offsets(lens, DEV)
    cub = inputs.qsa_offsets([L // 4 for L in lens], DEV)
    k_hat = torch.empty(sum(L // 4 for L in lens), 128, dtype=torch.bfloat16, device=DEV)
    q = inputs.qsa_queries(len(lens), 76, DEV)
    q_pos = torch.tensor([L - 1 for L in lens], dtype=torch.int32, device=DEV)
    ws = gdn.qsa_index_workspace(len(lens), k_hat.shape[0])
    bi = torch.empty(len(lens), 512, dtype=torch.int32, device=DEV)
    bs = torch.empty(len(lens), 512, device=DEV)
    ti = torch.empty(len(lens), 2048, dtype=torch.int32, device=DEV)

    def call():
        gdn.gdn_qsa_compress(k, cu, cub, k_hat=k_hat)
        gdn.gdn_qsa_index_decode(q, q_pos, k_hat, cub, 512, workspace=ws, block_idx=bi,
                                 block_score=bs, token_idx=ti)

    call()
    torch.cuda.synchronize()
    want = [t.clone() for t in (k_hat, bi, bs, ti)]
    g = _capture(call)
    for _ in range(3):                            # the workspace must be clean each time
        for t in (k_hat, bi, bs, ti):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        for t, wt in zip((k_hat, bi, bs, ti), want):
            assert torch.equal(t, wt)
