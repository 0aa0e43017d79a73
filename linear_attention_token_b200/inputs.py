"""Seeded synthetic inputs for the gated delta rule workloads.

This module only draws random tensors with the shapes, dtypes and value
distributions of the five workloads; it holds none of the layer's arithmetic.
Both the CUDA path (tests, bench) and the CPU oracle (tests) take their inputs
from here, and nothing else is shared between them.

Recipe (same for every workload unless stated):
  q, k ~ N(0, 1), L2-normalised per (token, head) in fp32, then cast;
  v ~ N(0, 1), cast;
  g = -softplus(N(0, 1))  (so alpha = exp(g) lies in (0, 1), the decay range
      of the gated delta rule in "論文解説: Qwen3.8-Next の設計", section
      "GDNの中身", text under Eq. (1));
  beta = sigmoid(N(0, 1))  (write strength in (0, 1), same passage);
  S0 = 0, or N(0, 0.02) (standard deviation 0.02) where the workload says so.

Layouts (B folded into the token axis; sequences are delimited by cu_seqlens):
  q, k  [T_total, H_qk, dk]   v, out [T_total, H_v, dv]
  g, beta [T_total, H_v] fp32  S0, S_final [N, H_v, dk, dv] fp32 (dv contiguous)
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

BASE_SEED = 20260


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    seq_lens: tuple           # per-sequence token counts (prefill); () for decode
    H_qk: int
    H_v: int
    dk: int
    dv: int
    dtype: torch.dtype        # dtype of q, k, v, out
    s0_std: float = 0.0       # 0 -> S0 = 0
    g_mult: float = 1.0       # multiplier on g (slow decay for the long workload)
    decode_seqs: int = 0      # decode only: independent sequences per step
    decode_steps: int = 0     # decode only: consecutive single-token steps
    index: int = 0            # workload number; seeds derive from it

    @property
    def num_seqs(self) -> int:
        return self.decode_seqs if self.kind == "decode" else len(self.seq_lens)

    @property
    def tokens(self) -> int:
        if self.kind == "decode":
            return self.decode_seqs * self.decode_steps
        return int(sum(self.seq_lens))

    @property
    def dense(self) -> bool:
        """True when every sequence has the same length (a [B, T] batch)."""
        return len(set(self.seq_lens)) <= 1


def _varlen_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    gen = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen))


def workloads() -> list:
    """The five workloads, by index."""
    return [
        Workload("prefill_b1_t256_h2_d64_f32", "prefill", (256,), 2, 2, 64, 64,
                 torch.float32, index=0),
        Workload("prefill_b2_t4096_h16_d128_bf16", "prefill", (4096, 4096), 16, 16,
                 128, 128, torch.bfloat16, index=1),
        Workload("prefill_varlen8_u1024_32768_hqk8_hv16_d128_bf16", "prefill",
                 _varlen_lengths(BASE_SEED + 2, 8, 1024, 32768), 8, 16, 128, 128,
                 torch.bfloat16, s0_std=0.02, index=2),
        Workload("prefill_b1_t262144_h16_d128_bf16_slowdecay", "prefill", (262144,),
                 16, 16, 128, 128, torch.bfloat16, g_mult=0.1, index=3),
        Workload("decode_n256_steps128_h32_d128_bf16_f32state", "decode", (), 32, 32,
                 128, 128, torch.bfloat16, s0_std=0.02, decode_seqs=256,
                 decode_steps=128, index=4),
    ]


def get(index: int) -> Workload:
    return workloads()[index]


def small(name: str, seq_lens, H_qk: int, H_v: int, dk: int, dv: int,
          dtype=torch.float32, s0_std: float = 0.0, g_mult: float = 1.0,
          index: int = 100) -> Workload:
    """An ad-hoc prefill workload (tests use these for ragged and edge cases)."""
    return Workload(name, "prefill", tuple(int(x) for x in seq_lens), H_qk, H_v, dk, dv,
                    dtype, s0_std=s0_std, g_mult=g_mult, index=index)


def cu_seqlens_of(seq_lens) -> torch.Tensor:
    cu = [0]
    for n in seq_lens:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def draw(T: int, H_qk: int, H_v: int, dk: int, dv: int, dtype, seed: int,
         device="cpu", g_mult: float = 1.0, normalize_qk: bool = True) -> dict:
    """Draw q, k, v, g, beta for T tokens with the recipe in the module docstring."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    f32 = torch.float32
    q = torch.randn(T, H_qk, dk, generator=gen, device=dev, dtype=f32)
    k = torch.randn(T, H_qk, dk, generator=gen, device=dev, dtype=f32)
    v = torch.randn(T, H_v, dv, generator=gen, device=dev, dtype=f32)
    g = -torch.nn.functional.softplus(torch.randn(T, H_v, generator=gen, device=dev, dtype=f32))
    if g_mult != 1.0:
        g = g * g_mult
    beta = torch.sigmoid(torch.randn(T, H_v, generator=gen, device=dev, dtype=f32))
    if normalize_qk:
        q, k = _l2n(q), _l2n(k)
    return {"q": q.to(dtype).contiguous(), "k": k.to(dtype).contiguous(),
            "v": v.to(dtype).contiguous(), "g": g.contiguous(), "beta": beta.contiguous()}


def draw_state(N: int, H_v: int, dk: int, dv: int, std: float, seed: int,
               device="cpu") -> Optional[torch.Tensor]:
    if std == 0.0:
        return None
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    return (torch.randn(N, H_v, dk, dv, generator=gen, device=dev, dtype=torch.float32)
            * std).contiguous()


def prefill_inputs(w: Workload, device="cpu", seed: Optional[int] = None) -> dict:
    """All prefill inputs for workload ``w``; S0 is None when the workload starts from 0."""
    assert w.kind == "prefill"
    s = BASE_SEED + w.index if seed is None else seed
    x = draw(w.tokens, w.H_qk, w.H_v, w.dk, w.dv, w.dtype, s, device, w.g_mult)
    x["S0"] = draw_state(w.num_seqs, w.H_v, w.dk, w.dv, w.s0_std, s + 7, device)
    x["cu_seqlens"] = cu_seqlens_of(w.seq_lens).to(device)
    return x


def decode_state(w: Workload, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """Initial decode state [N, H_v, dk, dv] fp32 ~ N(0, s0_std)."""
    assert w.kind == "decode"
    s = BASE_SEED + w.index if seed is None else seed
    return draw_state(w.decode_seqs, w.H_v, w.dk, w.dv, w.s0_std, s + 7, device)


def decode_step_inputs(w: Workload, step: int, device="cpu", seed: Optional[int] = None) -> dict:
    """q, k, v, g, beta for decode step ``step`` (one token per sequence)."""
    assert w.kind == "decode"
    s = (BASE_SEED + w.index if seed is None else seed) + 1000 * step
    return draw(w.decode_seqs, w.H_qk, w.H_v, w.dk, w.dv, w.dtype, s, device, w.g_mult)


# ------------------------------------------------------------------ QSA indexer
# Recipe: indexer keys and query heads ~ N(0, 1), cast to bf16.  A block-cache row stands
# for the mean of 4 such keys after a rotation, i.e. an isotropic normal with standard
# deviation 1/2; caches drawn directly take that distribution.  Palette caches (tests of
# exact ties) repeat a few rows c * v (c = 1, 2, ...) for one drawn vector v.
QSA_DIM, QSA_HEADS, QSA_R = 128, 4, 4
QSA_SEED = BASE_SEED + 40


@dataclasses.dataclass(frozen=True)
class QsaWorkload:
    name: str
    ctx_lens: tuple           # tokens per sequence so far; the query is the last of them
    budget_blocks: int = 512  # 2048 tokens at 4 tokens per block
    index: int = 0

    @property
    def num_seqs(self) -> int:
        return len(self.ctx_lens)

    @property
    def blocks(self) -> tuple:
        return tuple(int(L) // QSA_R for L in self.ctx_lens)


def qsa_workloads() -> list:
    return [
        QsaWorkload("qsa_decode_n8_ctx1m_budget2048", (1 << 20,) * 8, 512, index=0),
        QsaWorkload("qsa_decode_n5_ragged_budget2048", (70001, 8191, 4096, 3, 2052), 512,
                    index=1),
    ]


def qsa_keys(T: int, seed: int, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return torch.randn(T, QSA_DIM, generator=gen, device=device).to(torch.bfloat16).contiguous()


def qsa_queries(N: int, seed: int, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return (torch.randn(N, QSA_HEADS, QSA_DIM, generator=gen, device=device)
            .to(torch.bfloat16).contiguous())


def qsa_multi_queries(N: int, T: int, seed: int, device="cpu") -> torch.Tensor:
    """T consecutive query tokens per sequence: [N, T, 4, 128] bf16 ~ N(0, 1)."""
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return (torch.randn(N, T, QSA_HEADS, QSA_DIM, generator=gen, device=device)
            .to(torch.bfloat16).contiguous())


def qsa_cache(total_blocks: int, seed: int, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return ((torch.randn(total_blocks, QSA_DIM, generator=gen, device=device) * 0.5)
            .to(torch.bfloat16).contiguous())


def qsa_palette_cache(total_blocks: int, n_distinct: int, seed: int, device="cpu") -> torch.Tensor:
    """Rows c * v with c drawn from 1..n_distinct per row (exact ties inside each c)."""
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    v = torch.randn(QSA_DIM, generator=gen, device=device) * 0.5
    c = torch.randint(1, n_distinct + 1, (total_blocks, 1), generator=gen, device=device)
    return (c.to(torch.float32) * v).to(torch.bfloat16).contiguous()


def qsa_offsets(counts, device="cpu") -> torch.Tensor:
    return cu_seqlens_of(counts).to(device)


def qsa_decode_inputs(w: QsaWorkload, device="cpu", seed: Optional[int] = None) -> dict:
    """q [N, 4, 128], q_pos [N] (the last token of each sequence), the block cache and its
    row offsets."""
    s = QSA_SEED + w.index if seed is None else seed
    blocks = w.blocks
    return {
        "q": qsa_queries(w.num_seqs, s, device),
        "q_pos": torch.tensor([max(0, L - 1) for L in w.ctx_lens], dtype=torch.int32,
                              device=device),
        "k_hat": qsa_cache(int(sum(blocks)), s + 1, device),
        "cu_blocks": qsa_offsets(blocks, device),
    }
