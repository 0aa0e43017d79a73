"""Chunked prefill (gdn_prefill) against the CPU oracle, element by element.

The oracle is the token-by-token recurrence of Eq. (1) ("論文解説: Qwen3.8-Next の
設計", section "GDNの中身") in fp64 on the same (bf16-rounded) inputs; the chunked
kernels must match it within 1e-4 (fp32 inputs) or 2e-2 (bf16 inputs), measured as
max|x - ref| / max|ref| on the outputs and on the final state separately.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
from parity import TOL, err, oracle_prefill

pytestmark = pytest.mark.gpu

CC = gdn.GDN_FLAG_FORCE_CUDA_CORE


def run(x, flags=0, scale=1.0, dense_B=None):
    """Call gdn_prefill on the tensors in x (varlen form, or a dense [B, T] view)."""
    if dense_B is not None:
        B = dense_B
        T = x["q"].shape[0] // B
        view = lambda t: t.view(B, T, *t.shape[1:])
        o, S = gdn.gdn_prefill(view(x["q"]), view(x["k"]), view(x["v"]), view(x["g"]),
                               view(x["beta"]), x.get("S0"), None, scale=scale, flags=flags)
        o = o.view(B * T, *o.shape[2:])
    else:
        o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x.get("S0"),
                               x["cu_seqlens"], scale=scale, flags=flags)
    torch.cuda.synchronize()
    return o, S


def case(lens, H_qk, H_v, dk, dv, dtype, s0_std=0.0, seed=1, g_mult=1.0, normalize=True):
    w = inputs.small("t", lens, H_qk, H_v, dk, dv, dtype, s0_std=s0_std, g_mult=g_mult)
    x = inputs.draw(w.tokens, H_qk, H_v, dk, dv, dtype, seed, "cuda", g_mult, normalize)
    x["S0"] = inputs.draw_state(len(lens), H_v, dk, dv, s0_std, seed + 3, "cuda")
    x["cu_seqlens"] = inputs.cu_seqlens_of(lens).cuda()
    return x


def check(x, o, S, dtype, **kw):
    o_ref, S_ref = oracle_prefill(x, **kw)
    eo, es = err(o, o_ref), err(S, S_ref)
    assert eo < TOL[dtype], f"out err {eo:.3e}"
    assert es < TOL[dtype], f"state err {es:.3e}"
    return eo, es


# ------------------------------------------------------------------ workload 0
def test_workload0_fp32_full():
    """B=1, T=256, H=2, dk=dv=64, fp32, S0=0: every output and the final state."""
    w = inputs.get(0)
    x = {k: (v.cuda() if v is not None else None) for k, v in inputs.prefill_inputs(w).items()}
    o, S = run(x, dense_B=1)
    check(x, o, S, torch.float32)


# ---------------------------------------------------------------- edge shapes
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 1000])
@pytest.mark.parametrize("dtype,flags", [(torch.float32, 0), (torch.bfloat16, 0),
                                         (torch.bfloat16, CC)])
def test_dense_lengths(T, dtype, flags):
    x = case([T, T], 2, 2, 128, 128, dtype, s0_std=0.1, seed=T)
    o, S = run(x, flags=flags, dense_B=2)
    check(x, o, S, dtype)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_head_dims(dk, dv, dtype):
    x = case([130, 70], 1, 2, dk, dv, dtype, s0_std=0.1, seed=dk + dv)
    o, S = run(x)
    check(x, o, S, dtype)


@pytest.mark.parametrize("dtype,flags", [(torch.float32, 0), (torch.bfloat16, 0),
                                         (torch.bfloat16, CC)])
def test_varlen_gva_ragged(dtype, flags):
    lens = [1, 0, 64, 65, 129, 300, 2, 191]
    x = case(lens, 2, 4, 128, 128, dtype, s0_std=0.05, seed=11)
    o, S = run(x, flags=flags)
    check(x, o, S, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_l2norm_flag_and_scale(dtype):
    x = case([200, 77], 2, 2, 128, 128, dtype, s0_std=0.05, seed=12, normalize=False)
    o, S = run(x, flags=gdn.GDN_FLAG_QK_L2NORM, scale=0.125)
    check(x, o, S, dtype, l2norm=True, scale=0.125)


def test_strong_decay_stays_finite():
    """g ~ -3 softplus(N(0,1)): in-chunk cumulative decay reaches ~ -150 within a chunk."""
    x = case([512], 2, 2, 128, 128, torch.bfloat16, seed=13, g_mult=3.0)
    o, S = run(x)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    check(x, o, S, torch.bfloat16)


def test_empty_input_copies_state():
    x = case([0, 0], 1, 2, 128, 128, torch.bfloat16, s0_std=0.1, seed=14)
    o, S = run(x)
    assert torch.equal(S, x["S0"])


# ------------------------------------------------------ segmented (sequence-parallel)
@pytest.fixture
def segments():
    """Force the sequence-parallel schedule with a given segment length for one test."""
    def set_(tokens):
        gdn.gdn_set_prefill_segment_tokens(tokens)
    yield set_
    gdn.gdn_set_prefill_segment_tokens(0)


@pytest.mark.parametrize("seg", [64, 128, 192])
def test_segmented_varlen_gva_ragged(segments, seg):
    """Segments of `seg` tokens: the transfer pass, the scan and the output pass against
    the oracle; lengths cut segments at, before and after chunk edges, and include
    sequences shorter than one segment (a single unit) and empty ones."""
    segments(seg)
    lens = [1, 0, 64, 65, 129, 300, 2, 191, 640]
    x = case(lens, 2, 4, 128, 128, torch.bfloat16, s0_std=0.05, seed=21 + seg)
    o, S = run(x)
    check(x, o, S, torch.bfloat16)


@pytest.mark.parametrize("seg", [64, 256])
def test_segmented_dense(segments, seg):
    """Dense batch, segments per sequence from the batch shape (no unit table)."""
    segments(seg)
    x = case([1000, 1000, 1000], 1, 2, 128, 128, torch.bfloat16, s0_std=0.1, seed=31 + seg)
    o, S = run(x, dense_B=3)
    check(x, o, S, torch.bfloat16)


def test_segmented_strong_decay_and_l2norm(segments):
    segments(128)
    x = case([700, 333], 2, 2, 128, 128, torch.bfloat16, s0_std=0.05, seed=41, g_mult=3.0,
             normalize=False)
    o, S = run(x, flags=gdn.GDN_FLAG_QK_L2NORM, scale=0.5)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    check(x, o, S, torch.bfloat16, l2norm=True, scale=0.5)


@pytest.mark.parametrize("lens", [[1, 0, 64, 65, 129, 300, 2, 191], [1000, 1000]])
def test_cluster_kernel(segments, lens):
    """The four-CTA cluster kernel (value columns split four ways, each chunk prepared by
    one CTA of the cluster) on ragged varlen input with grouped heads and S0."""
    segments(-2)
    x = case(lens, 2, 4, 128, 128, torch.bfloat16, s0_std=0.05, seed=61 + len(lens))
    o, S = run(x)
    check(x, o, S, torch.bfloat16)


def test_schedules_agree(segments):
    """The one-unit and segmented schedules give the same results up to rounding."""
    x = case([900, 450], 2, 2, 128, 128, torch.bfloat16, s0_std=0.05, seed=51)
    segments(-1)
    o1, S1 = run(x)
    segments(192)
    o2, S2 = run(x)
    segments(-2)
    o3, S3 = run(x)
    assert err(o2, o1) < 1e-2 and err(S2, S1) < 1e-2
    assert err(o3, o1) < 1e-2 and err(S3, S1) < 1e-2


# ---------------------------------------------------------- full-size workloads
def _full(idx):
    w = inputs.get(idx)
    x = inputs.prefill_inputs(w, device="cuda")
    return w, x


def test_workload1_full():
    """B=2, T=4096, H=16, d=128, bf16: all 32 (sequence, head) pairs against the oracle."""
    w, x = _full(1)
    o, S = run(x, dense_B=2)
    check(x, o, S, torch.bfloat16)


def test_workload2_varlen_sampled():
    """8 packed sequences (seeded lengths in [1024, 32768]), 8 q/k heads shared by 16 value
    heads, S0 ~ N(0, 0.02): three value heads of every sequence against the oracle."""
    w, x = _full(2)
    o, S = run(x)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    heads = [0, 7, 15]
    o_ref, S_ref = oracle_prefill(x, heads=heads)
    assert err(o[:, heads], o_ref) < TOL[torch.bfloat16]
    assert err(S[:, heads], S_ref) < TOL[torch.bfloat16]


def test_workload3_long_sampled():
    """B=1, T=262144, H=16, slow decay: two heads over the whole sequence against the oracle."""
    w, x = _full(3)
    o, S = run(x, dense_B=1)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    heads = [3, 12]
    o_ref, S_ref = oracle_prefill(x, heads=heads)
    assert err(o[:, heads], o_ref) < TOL[torch.bfloat16]
    assert err(S[:, heads], S_ref) < TOL[torch.bfloat16]
