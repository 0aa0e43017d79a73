"""bench.py's algorithmic counts and its traffic keying, on the CPU.

The roofline fractions bench.py reports divide these counts by measured times, so they are
checked against figures derived independently of the code: the hot-path table's FLOP and
byte counts for the workloads, and the QSA call's bytes from its definition.
"""
from __future__ import annotations

import importlib.util
import os

import pytest

from linear_attention_token_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_prefill_flops_per_token_head(bench):
    # 2 [C (3 dk + 2 dv) + 3 dk dv] at C = 64
    assert bench.prefill_flops_per_token_head(128, 128) == 180_224
    assert bench.prefill_flops_per_token_head(64, 64) == 65_536


def test_midsize_workload_counts(bench):
    w = inputs.get(1)
    flops = bench.prefill_flops_per_token_head(w.dk, w.dv) * w.tokens * w.H_v
    assert abs(flops - 23.62e9) < 0.01e9
    # q, k, v, out bf16 (16,384 B per token), g and beta fp32, S_final once (S0 = 0)
    assert bench.prefill_bytes(w) == 8192 * 16_384 + 8192 * 16 * 8 + 2 * 16 * 128 * 128 * 4


def test_decode_bytes_per_step(bench):
    w = inputs.get(4)
    b = bench.decode_bytes_per_step(w)
    assert abs(b / 1e6 - 1082.2) < 0.05
    # the state read and written once dominates: 256 x 32 heads x 64 KB x 2
    assert b > 256 * 32 * 128 * 128 * 4 * 2


def test_decode_multi_bytes(bench):
    w = inputs.get(4)
    one = bench.decode_multi_bytes_per_call(w, 1)
    assert one == bench.decode_bytes_per_step(w)
    four = bench.decode_multi_bytes_per_call(w, 4)
    assert four - one == 3 * (one - 256 * 32 * 128 * 128 * 4 * 2)


def test_qsa_index_bytes(bench):
    wq = inputs.qsa_workloads()[0]
    b = bench.qsa_index_bytes(wq, sum(wq.blocks))
    # 8 x 262,144 cache rows of 256 B, queries and positions, 512 kept blocks out
    assert b == 8 * 262_144 * 256 + 8 * (4 * 128 * 2 + 4) + 8 * 512 * (4 + 4 + 16)
    assert abs(b / 1e6 - 537.0) < 0.1


def test_traffic_key_ignores_comments_only(bench, tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void f(int *p) {\n  p[0] = 1;  /* store */\n}\n")
    k0 = bench.source_code_key(str(src))
    src.write_text("// another header\n\n__global__ void f(int *p) {\n    p[0] = 1;\n}\n")
    assert bench.source_code_key(str(src)) == k0
    src.write_text("__global__ void f(int *p) {\n  p[0] = 2;\n}\n")
    assert bench.source_code_key(str(src)) != k0


def test_traffic_file_is_well_formed():
    """Each entry: kernel key, 16 hex digits of the code key, bytes per launch.  (An entry
    whose code key no longer matches the source is allowed: bench.py then reports null.)"""
    known = {"prefill_long", "prefill", "decode", "decode_multi", "backward", "qsa_score",
             "qsa_compress", "qsa_score_t4"}
    n = 0
    for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        key, code, nbytes = line.split()[:3]
        assert key in known, key
        assert len(code) == 16 and int(code, 16) >= 0
        assert int(nbytes) > 0
        n += 1
    assert n >= len(known) - 1          # every kernel but possibly the newest entry


def test_long_context_workload_counts(bench):
    """The headline workload: 262,144 tokens x 16 heads; 755.9 GFLOP and 4.33 GB."""
    w = inputs.get(3)
    flops = bench.prefill_flops_per_token_head(w.dk, w.dv) * w.tokens * w.H_v
    assert abs(flops - 755.9e9) < 0.1e9
    assert bench.prefill_bytes(w) == 262_144 * 8192 * 2 + 262_144 * 16 * 8 + 16 * 128 * 128 * 4


def test_prefill_args_dense_and_varlen(bench):
    # dense workloads run as a [B, T] batch; the varlen one passes cu_seqlens and S0
    for idx, varlen in ((1, False), (3, False), (2, True)):
        w = inputs.get(idx)
        x = {n: None for n in ("q", "k", "v", "g", "beta", "S0")}
        x["cu_seqlens"] = "offsets"
        if not varlen:
            B, T = len(w.seq_lens), w.seq_lens[0]
            import torch
            x = {n: torch.zeros(B * T, 1) for n in ("q", "k", "v", "g", "beta")}
        args, N = bench.prefill_args(x, w)
        assert N == len(w.seq_lens)
        assert (args[6] is not None) == varlen
