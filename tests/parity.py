"""Shared helpers for the GPU parity tests: run the oracle on the very inputs the
CUDA path reads, and measure the error the way the tolerances are stated.

err(x, ref) = max|x - ref| / max|ref|, computed separately for the outputs and the
final state.  Limits (stated for the gated delta rule workloads): 1e-4 with fp32
inputs, 2e-2 with bf16 inputs (fp32 state in both cases).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = ref.detach().double().cpu().numpy() if hasattr(ref, "detach") else np.asarray(ref, np.float64)
    if x.size == 0:
        return 0.0
    den = np.max(np.abs(ref))
    num = np.max(np.abs(x - ref))
    return float(num / den) if den > 0 else float(num)


def oracle_prefill(x: dict, scale=1.0, l2norm=False, heads=None, seqs=None, threads=0):
    """Oracle outputs for the tensors in ``x`` (as read by the GPU: bf16 values upcast).

    heads / seqs restrict the run to a subset (sampled checks at full size); the
    returned arrays then cover only those value heads / sequences, in order.
    """
    q, k, v, g, beta = (x[n] for n in ("q", "k", "v", "g", "beta"))
    S0 = x.get("S0")
    cu = x["cu_seqlens"].cpu().numpy().astype(np.int64)
    H_v = v.shape[-2]
    H_qk = q.shape[-2]
    group = H_v // H_qk
    if seqs is not None:
        parts = [slice(int(cu[n]), int(cu[n + 1])) for n in seqs]
        pick = lambda t: torch.cat([t[p] for p in parts]) if len(parts) else t[:0]
        q, k, v, g, beta = (pick(t) for t in (q, k, v, g, beta))
        lens = [int(cu[n + 1] - cu[n]) for n in seqs]
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        if S0 is not None:
            S0 = S0[list(seqs)]
    if heads is not None:
        heads = list(heads)
        # run each value head with its own q/k head (group of 1)
        q = q[:, [h // group for h in heads]]
        k = k[:, [h // group for h in heads]]
        v, g, beta = v[:, heads], g[:, heads], beta[:, heads]
        if S0 is not None:
            S0 = S0[:, heads]
    o, S = oracle.recurrent(q, k, v, g, beta, S0=S0, cu_seqlens=cu, scale=scale, l2norm=l2norm,
                            threads=threads)
    return o, S


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
