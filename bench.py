#!/usr/bin/env python
"""Throughput of the gated delta rule (Gated DeltaNet token mixing) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line.  A step is one gdn_prefill call over the long-context prefill
workload (B=1, T=262,144, H=16, dk=dv=128, bf16 q/k/v, fp32 g/beta/state, slow decay
g = -0.1 softplus(N(0,1)), S0=0); `value` is whole-job prefill tokens/s with the inputs
resident in HBM.  The same line carries, with short keys so that it stays compact:
"roofline" of that call, "e2e" (the same call through the C ABI from pinned host memory,
copies inside the timed region), "decode" (256 sequences x 128 single-token steps, H=32,
fp32 state ~ N(0, 0.02)), "cpu_baseline" (the oracle on this host's cores, on a prefix of
the workload), and "sections": the mid-size and varlen prefill workloads, multi-token
decode, the backward pass and the QSA compressed indexer.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on the
launching stream; a 256 MB buffer is written between prefill steps (outside the events)
so no step starts with inputs in the 126 MB L2 (the long-context inputs are 4.3 GB in any
case).  The decode state (537 MB) is larger than L2.  With N > 1 (torchrun) every rank
runs its own replica of the workload (the layer has no cross-GPU exchange), the job time
is the max over ranks and `value` counts all ranks' tokens.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_token_b200 import inputs  # noqa: E402

METRIC = "GDN prefill tokens/s and decode tokens/s on 1 B200; % of tensor/HBM roofline"
PREFILL_W = 3          # headline: the long-context prefill
MID_W, VARLEN_W = 1, 2
DECODE_W = 4
CHUNK = 64


# ----------------------------------------------------------------- algorithmic counts
def prefill_flops_per_token_head(dk: int, dv: int, C: int = CHUNK) -> int:
    """The chunked method's contractions at tile shape, per token per value head:
    [K;Q]K^T (2 C dk), K^T T'^T / V^T T''^T (C dk + C dv), W S and Q S (2 dk dv),
    (P U) (C dv) and the state update K~^T U (dk dv), times 2 flops per MAC."""
    return 2 * (C * (3 * dk + 2 * dv) + 3 * dk * dv)


def prefill_bytes(w) -> int:
    """q/k/v/out once in the I/O dtype, g and beta in fp32, S0 and S_final once."""
    e = torch.tensor([], dtype=w.dtype).element_size()
    T = w.tokens
    b = T * (2 * w.H_qk * w.dk + 2 * w.H_v * w.dv) * e + T * w.H_v * 8
    b += w.num_seqs * w.H_v * w.dk * w.dv * 4 * (2 if w.s0_std else 1)
    return b


def decode_bytes_per_step(w) -> int:
    e = torch.tensor([], dtype=w.dtype).element_size()
    N = w.decode_seqs
    return (N * w.H_v * w.dk * w.dv * 4 * 2 + N * (2 * w.H_qk * w.dk + 2 * w.H_v * w.dv) * e
            + N * w.H_v * 8)


VERIFY_T = 4      # tokens per gdn_decode_multi call (e.g. three drafted tokens + one)


def decode_multi_bytes_per_call(w, T: int) -> int:
    """Algorithmic bytes of one multi-token call: the state read and written once, and T
    tokens' q, k, v, out, g, beta."""
    e = torch.tensor([], dtype=w.dtype).element_size()
    N = w.decode_seqs
    return (N * w.H_v * w.dk * w.dv * 4 * 2
            + T * (N * (2 * w.H_qk * w.dk + 2 * w.H_v * w.dv) * e + N * w.H_v * 8))


def qsa_index_bytes(wq, blocks: int) -> int:
    """Algorithmic bytes of one indexer call: every cached block row read once (128 bf16),
    the queries (4 x 128 bf16 per sequence) and positions read once, the kept blocks, their
    scores and tokens written once."""
    N, K = wq.num_seqs, wq.budget_blocks
    return blocks * 256 + N * (4 * 128 * 2 + 4) + N * K * (4 + 4 + 4 * 4)


def decode_flops_per_step(w) -> int:
    # a = S^T k, b = S^T q, S <- alpha S + k u^T: 3 MACs per state element
    return 2 * 3 * w.decode_seqs * w.H_v * w.dk * w.dv


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_code_key(source_file: str) -> str:
    """sha256 (first 16 hex digits) of a CUDA source with its comments and whitespace
    removed: a comment-only edit keeps the key, any change to the code changes it."""
    text = open(source_file).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()[:16]


def profiled_traffic(kernel_key: str, source_file: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel's code as it is now (source_code_key of the .cu file recorded in the summary)."""
    summary = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(summary):
        return None
    sha = source_code_key(source_file)
    for line in open(summary):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_key and parts[1] == sha:
            return int(float(parts[2]))
    return None


# -------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), p[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        load = [r for r in rows if r[0] > 0.5 * r[1]] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, x in enumerate(r[2]) if x == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------- our arm
def flush_l2(buf):
    buf.add_(1)


def prefill_args(x, w):
    """The gdn_prefill arguments for workload w: a dense [B, T] view, or varlen."""
    if len(set(w.seq_lens)) == 1 and not w.s0_std:
        B, T = len(w.seq_lens), w.seq_lens[0]
        view = lambda t: t.view(B, T, *t.shape[1:])
        return [view(x[n]) for n in ("q", "k", "v", "g", "beta")] + [None, None], B
    return [x[n] for n in ("q", "k", "v", "g", "beta")] + [x["S0"], x["cu_seqlens"]], len(w.seq_lens)


def time_prefill(gdn, x, w, steps, warmup, stream, flush):
    args, N = prefill_args(x, w)
    out = torch.empty_like(args[2])
    S_final = torch.empty(N, w.H_v, w.dk, w.dv, dtype=torch.float32, device=out.device)
    ws = gdn.prefill_workspace(N, w.tokens, w.H_v, w.dk, w.dv, out.device)
    sched = gdn.gdn_prefill_schedule(N, w.tokens, w.H_v, w.dk, w.dv, w.dtype,
                                     varlen=args[6] is not None, workspace_bytes=ws.numel())
    call = lambda: gdn.gdn_prefill(*args, out=out, S_final=S_final, workspace=ws, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush_l2(flush)
            call()
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush_l2(flush)
            a.record(stream)
            call()
            b.record(stream)
    stream.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    status = gdn.gdn_get_device_error(ws, stream)
    del ws, out, S_final
    return times, status, sched


def time_prefill_e2e(gdn, w, steps, warmup, stream, device):
    """Through the public API with HOST buffers: every step copies its inputs in from pinned
    host memory, runs the prefill and copies its result (outputs and final state) back.
    Consecutive steps alternate between two streams and two device buffer sets, so one
    step's copy out overlaps the next step's copy in (separate copy engines) and compute;
    the events bracket all `steps` steps."""
    B, T = len(w.seq_lens), w.seq_lens[0]
    xh = inputs.prefill_inputs(w, device="cpu")
    host = {n: xh[n].view(B, T, *xh[n].shape[1:]).pin_memory() for n in ("q", "k", "v", "g", "beta")}
    del xh
    streams = [stream, torch.cuda.Stream(device)]
    sets = []
    for _ in range(2):
        sets.append({
            "dev": {n: torch.empty_like(t, device=device) for n, t in host.items()},
            "out_h": torch.empty(host["v"].shape, dtype=w.dtype).pin_memory(),
            "S_h": torch.empty(B, w.H_v, w.dk, w.dv, dtype=torch.float32).pin_memory(),
            "out_d": torch.empty(host["v"].shape, dtype=w.dtype, device=device),
            "S_d": torch.empty(B, w.H_v, w.dk, w.dv, dtype=torch.float32, device=device),
            "ws": gdn.prefill_workspace(B, w.tokens, w.H_v, w.dk, w.dv, device)})
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sets[0]["out_h"].numel() * sets[0]["out_h"].element_size() + sets[0]["S_h"].numel() * 4

    def step(i):
        st, b = streams[i % 2], sets[i % 2]
        with torch.cuda.stream(st):
            for n in host:
                b["dev"][n].copy_(host[n], non_blocking=True)
            gdn.gdn_prefill(b["dev"]["q"], b["dev"]["k"], b["dev"]["v"], b["dev"]["g"],
                            b["dev"]["beta"], None, None, out=b["out_d"], S_final=b["S_d"],
                            workspace=b["ws"], stream=st)
            b["out_h"].copy_(b["out_d"], non_blocking=True)
            b["S_h"].copy_(b["S_d"], non_blocking=True)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    other_done = torch.cuda.Event()
    start.record(streams[0])
    streams[1].wait_event(start)
    for i in range(steps):
        step(i)
    other_done.record(streams[1])
    streams[0].wait_event(other_done)
    end.record(streams[0])
    torch.cuda.synchronize(device)
    per_step = start.elapsed_time(end) / steps
    del sets, host
    torch.cuda.empty_cache()
    return [per_step], h2d, d2h


def time_decode(gdn, w, passes, warmup, stream, device):
    """`passes` timed passes of all decode steps (each pass: decode_steps launches)."""
    S = inputs.decode_state(w, device)
    xs = [inputs.decode_step_inputs(w, s, device) for s in range(w.decode_steps)]
    outs = [torch.empty_like(x["v"]) for x in xs]

    def one_pass():
        for x, o in zip(xs, outs):
            gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out=o, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_pass()
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(passes)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            a.record(stream)
            one_pass()
            b.record(stream)
    stream.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_decode_multi(gdn, w, T, passes, warmup, stream, device):
    """The decode workload's token stream, T consecutive tokens per gdn_decode_multi call
    (decode_steps / T calls per pass, every token committed)."""
    S = inputs.decode_state(w, device)
    steps = [inputs.decode_step_inputs(w, s, device) for s in range(w.decode_steps)]
    xs = [{n: torch.stack([steps[j * T + t][n] for t in range(T)], dim=1).contiguous()
           for n in ("q", "k", "v", "g", "beta")} for j in range(w.decode_steps // T)]
    del steps
    outs = [torch.empty_like(x["v"]) for x in xs]

    def one_pass():
        for x, o in zip(xs, outs):
            gdn.gdn_decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out=o, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_pass()
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(passes)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            a.record(stream)
            one_pass()
            b.record(stream)
    stream.synchronize()
    return [a.elapsed_time(b) for a, b in evs], len(xs)


def time_backward(gdn, x, w, steps, warmup, stream):
    """gdn_backward on the mid-size prefill workload (d_out random, no dS_final), device-timed."""
    B, T = len(w.seq_lens), w.seq_lens[0]
    view = lambda t: t.view(B, T, *t.shape[1:])
    gen = torch.Generator(device="cpu").manual_seed(inputs.BASE_SEED + 99)
    d_out = torch.randn(x["v"].shape, generator=gen).to(w.dtype).to(x["v"].device)
    args = [view(x[n]) for n in ("q", "k", "v", "g", "beta")] + [view(d_out)]
    ws = torch.empty(int(gdn.lib().gdn_backward_workspace_size(B, B * T, w.H_v, w.dk, w.dv)),
                     dtype=torch.uint8, device=d_out.device)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            gdn.gdn_backward(*args, workspace=ws, stream=stream)
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            a.record(stream)
            gdn.gdn_backward(*args, workspace=ws, stream=stream)
            b.record(stream)
    stream.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_qsa(gdn, wq, steps, warmup, stream, device):
    """The QSA indexer on its decode workload (8 sequences x 1,048,576 cached tokens =
    262,144 blocks each, budget 512 blocks): each timed call is one gdn_qsa_index_decode
    (score, threshold, collect and finish kernels).  The 512 MB block cache is larger than
    L2, so no flush is needed between calls.  Then gdn_qsa_compress over the same
    sequences' 8,388,608 raw keys (2.1 GB in, 0.5 GB out)."""
    x = inputs.qsa_decode_inputs(wq, device)
    N, nb = wq.num_seqs, x["k_hat"].shape[0]
    ws = gdn.qsa_index_workspace(N, nb, device)
    bi = torch.empty(N, wq.budget_blocks, dtype=torch.int32, device=device)
    bs = torch.empty(N, wq.budget_blocks, dtype=torch.float32, device=device)
    ti = torch.empty(N, 4 * wq.budget_blocks, dtype=torch.int32, device=device)

    def call():
        gdn.gdn_qsa_index_decode(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"],
                                 wq.budget_blocks, workspace=ws, block_idx=bi, block_score=bs,
                                 token_idx=ti, stream=stream)

    def timed(fn, n, warm):
        with torch.cuda.stream(stream):
            for _ in range(warm):
                fn()
        stream.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
        stream.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    itimes = timed(call, steps, warmup)
    # the same caches with 4 query tokens per sequence (drafted tokens checked together)
    Tq = 4
    qm = inputs.qsa_multi_queries(N, Tq, inputs.QSA_SEED + 60, device)
    qm_pos = torch.tensor([L - Tq for L in wq.ctx_lens], dtype=torch.int32, device=device)
    wsm = gdn.qsa_index_multi_workspace(N, nb, Tq, device)
    bim = torch.empty(N, Tq, wq.budget_blocks, dtype=torch.int32, device=device)
    bsm = torch.empty(N, Tq, wq.budget_blocks, dtype=torch.float32, device=device)
    tim = torch.empty(N, Tq, 4 * wq.budget_blocks, dtype=torch.int32, device=device)
    mtimes = timed(lambda: gdn.gdn_qsa_index_multi(qm, qm_pos, x["k_hat"], x["cu_blocks"],
                                                   wq.budget_blocks, workspace=wsm,
                                                   block_idx=bim, block_score=bsm,
                                                   token_idx=tim, stream=stream),
                   steps, warmup)
    del wsm
    T = sum(wq.ctx_lens)
    k = inputs.qsa_keys(T, inputs.QSA_SEED + 50, device)
    cu = inputs.qsa_offsets(wq.ctx_lens, device)
    k_hat = torch.empty(nb, 128, dtype=torch.bfloat16, device=device)
    ctimes = timed(lambda: gdn.gdn_qsa_compress(k, cu, x["cu_blocks"], k_hat=k_hat,
                                                stream=stream), max(1, min(steps, 5)), 1)
    del k, k_hat
    return itimes, ctimes, nb, T, mtimes


def cpu_baseline_qsa(wq, seqs=2):
    """The oracle's indexer (float64 numpy, Python ranking) on `seqs` of the workload's
    queries, timed on this host."""
    from oracle import qsa as oq
    x = inputs.qsa_decode_inputs(wq, "cpu")
    cb = x["cu_blocks"].numpy()
    q = x["q"][:seqs].float().numpy()
    kh = x["k_hat"][:int(cb[seqs])].float().numpy()
    t0 = time.perf_counter()
    oq.index_decode(q, x["q_pos"][:seqs].numpy(), kh, cb[:seqs + 1], wq.budget_blocks)
    dt = time.perf_counter() - t0
    return {"value": seqs / dt, "unit": "queries/s", "cores": 1, "kind": "oracle",
            "sample": f"{seqs} of the {wq.num_seqs} queries (262,144 blocks each), float64 "
                      f"numpy scores and Python ranking, one thread"}


def cpu_baseline_prefill(w, max_tokens=None):
    """The oracle (float variant, all host cores) on the prefill workload, timed; with
    max_tokens, on the first max_tokens // N tokens of every sequence (the sequential
    recurrence costs the same per token anywhere in a sequence, so tokens/s from a prefix
    is the whole workload's rate)."""
    import oracle
    x = inputs.prefill_inputs(w, device="cpu")
    cu = x["cu_seqlens"]
    if max_tokens is not None and w.tokens > max_tokens:
        lens = [min(n, max_tokens // len(w.seq_lens)) for n in w.seq_lens]
        parts = [slice(int(cu[i]), int(cu[i]) + lens[i]) for i in range(len(lens))]
        pick = lambda t: torch.cat([t[p] for p in parts])
        x = {n: pick(x[n]) for n in ("q", "k", "v", "g", "beta")} | {"S0": x["S0"]}
        cu = inputs.cu_seqlens_of(lens)
    q, k, v, g, beta = (x[n].float().numpy() for n in ("q", "k", "v", "g", "beta"))
    S0 = None if x["S0"] is None else x["S0"].numpy()
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v, g, beta, S0=S0, cu_seqlens=cu.numpy(), precision="f32",
                     threads=threads)
    dt = time.perf_counter() - t0
    ntok = int(cu[-1])
    return {"value": ntok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"first {ntok} of {w.tokens} tokens x {w.H_v} heads of {w.name} "
                      f"(sequential fp32 recurrence, {threads} threads over (sequence, head))"}


def cpu_baseline_decode(w, steps=2):
    import oracle
    S = inputs.decode_state(w, "cpu").numpy()
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    for s in range(steps):
        x = inputs.decode_step_inputs(w, s, "cpu")
        q, k, v, g, beta = (x[n].float().numpy() for n in ("q", "k", "v", "g", "beta"))
        import numpy as np
        cu = np.arange(w.decode_seqs + 1, dtype=np.int64)
        _, S = oracle.recurrent(q, k, v, g, beta, S0=S, cu_seqlens=cu, precision="f32",
                                threads=threads)
    dt = time.perf_counter() - t0
    return {"value": steps * w.decode_seqs / dt, "unit": "tokens/s", "cores": threads,
            "kind": "oracle", "seconds": dt,
            "sample": f"{steps} of {w.decode_steps} decode steps x {w.decode_seqs} sequences x "
                      f"{w.H_v} heads of {w.name}"}


def dist_init(backend=None, timeout_s: float = 120.0):
    """One process per GPU under torchrun (RANK / WORLD_SIZE / MASTER_* from the env):
    NCCL on GPUs; gloo when there is no GPU (the CPU tests of this plumbing).  The
    ranks are replicas: nothing but the barrier and the max-over-ranks timing crosses
    between them."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    kwargs = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kwargs["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kwargs)
    return rank, world, local


def _device_sync():
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    _device_sync()


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas: every rank's tokens over the slowest
    rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def qsa_workload(args):
    w = inputs.qsa_workloads()[0]
    if args.qsa_seqs != w.num_seqs:
        w = inputs.QsaWorkload(f"qsa_decode_n{args.qsa_seqs}_ctx1m_budget2048",
                               (w.ctx_lens[0],) * args.qsa_seqs, w.budget_blocks, w.index)
    return w


def qsa_section(gdn, peaks, wq, qtimes, ctimes, q_blocks, q_tokens, world, mtimes):
    ms_qsa = max_over_ranks(sum(qtimes) / len(qtimes), world)
    ms_multi = max_over_ranks(sum(mtimes) / len(mtimes), world)
    multi_bytes = q_blocks * 256 + wq.num_seqs * 4 * (4 * 128 * 2 + 4) + \
        wq.num_seqs * 4 * wq.budget_blocks * (4 + 4 + 4 * 4)
    multi_gbs = multi_bytes / (ms_multi * 1e-3) / 1e9
    ms_cmp = max_over_ranks(sum(ctimes) / len(ctimes), world)
    qsa_bytes = qsa_index_bytes(wq, q_blocks)
    qsa_gbs = qsa_bytes / (ms_qsa * 1e-3) / 1e9
    cmp_bytes = q_tokens * 256 + q_blocks * 256
    cmp_gbs = cmp_bytes / (ms_cmp * 1e-3) / 1e9
    qsa_src = os.path.join(ROOT, "linear_attention_token_b200", "csrc", "qsa.cu")
    scale = wq.num_seqs / 8          # the traffic entries are per launch of the 8-sequence case

    def tr(key):
        t = profiled_traffic(key, qsa_src)
        return None if t is None else int(t * scale)

    return {
        "workload": wq.name, "value": world * wq.num_seqs / (ms_qsa * 1e-3),
        "unit": "queries/s", "ms_per_call": ms_qsa, "calls": len(qtimes),
        "budget_blocks": wq.budget_blocks, "cached_blocks": q_blocks,
        "roofline": {"bound": "hbm", "achieved": qsa_gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": qsa_gbs / peaks["hbm_gbs"],
                     "traffic": tr("qsa_score"),
                     "peak_source": f"{peaks['source']} copy bandwidth",
                     "algorithmic_bytes_per_launch": qsa_bytes,
                     "timed": "the whole gdn_qsa_index_decode call (score, collect and finish "
                              "kernels, calls back to back); the score kernel is the dominant one"},
        "multi_query": {
            "workload": f"{wq.name} with 4 query tokens per sequence (drafted tokens, each at "
                        f"its own position; one gdn_qsa_index_multi call)",
            "value": world * wq.num_seqs * 4 / (ms_multi * 1e-3), "unit": "queries/s",
            "ms_per_call": ms_multi, "calls": len(mtimes),
            "roofline": {"bound": "hbm", "achieved": multi_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": multi_gbs / peaks["hbm_gbs"],
                         "traffic": tr("qsa_score_t4"), "algorithmic_bytes_per_launch": multi_bytes,
                         "timed": "the whole call; the cache is read once for all 4 queries"}},
        "compress": {
            "workload": f"{wq.num_seqs} x {wq.ctx_lens[0]} raw keys -> {q_blocks} blocks",
            "value": world * q_tokens / (ms_cmp * 1e-3), "unit": "tokens/s",
            "ms_per_call": ms_cmp, "calls": len(ctimes),
            "roofline": {"bound": "hbm", "achieved": cmp_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": cmp_gbs / peaks["hbm_gbs"],
                         "traffic": tr("qsa_compress"),
                         "algorithmic_bytes_per_launch": cmp_bytes}},
    }


def run_qsa_only(args):
    """--section qsa: the QSA indexer and compression alone (one JSON line)."""
    rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import linear_attention_token_b200 as gdn
    gdn.lib()
    peaks = load_peaks()
    stream = torch.cuda.Stream(device)
    wq = qsa_workload(args)
    barrier(world)
    with ClockSampler(local) as clk:
        qtimes, ctimes, q_blocks, q_tokens, mtimes = time_qsa(gdn, wq, max(1, args.steps),
                                                              max(args.warmup, 1), stream, device)
        barrier(world)
    sec = qsa_section(gdn, peaks, wq, qtimes, ctimes, q_blocks, q_tokens, world, mtimes)
    line = {"metric": "QSA indexer queries/s on 1 B200; % of HBM roofline",
            "value": sec["value"], "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 1), "ms_per_step": sec["ms_per_call"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; block cache ~ N(0, 1/4), query heads ~ N(0, 1))",
            "config": {"workload": wq.name}, "qsa_indexer": sec,
            "gpu_launches": 3 * len(qtimes) + 3 * len(mtimes) + len(ctimes),
            "clocks": clk.summary()}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_prefill_only(args):
    """--section prefill: one prefill workload alone (one JSON line), optionally cut to its
    first --prefill-tokens tokens per sequence, so a profiler can capture a few launches on
    a small case of the same kernels."""
    import dataclasses
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import linear_attention_token_b200 as gdn
    gdn.lib()
    peaks = load_peaks()
    w = inputs.get(args.prefill_workload)
    if args.prefill_tokens:
        n = int(args.prefill_tokens)
        w = dataclasses.replace(w, name=f"{w.name}_first{n}",
                                seq_lens=tuple(min(n, L) for L in w.seq_lens))
    stream = torch.cuda.Stream(device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    x = inputs.prefill_inputs(w, device=device)
    gdn.gdn_set_prefill_segment_tokens(args.segment_tokens)
    with ClockSampler(0) as clk:
        times, status, sched = time_prefill(gdn, x, w, max(1, args.steps), max(args.warmup, 1),
                                            stream, flush)
    if status != 0:
        raise RuntimeError(f"device error after prefill: {gdn.gdn_status_string(status)}")
    ms = sum(times) / len(times)
    print(json.dumps({"metric": "GDN prefill tokens/s on 1 B200", "value": w.tokens / (ms * 1e-3),
                      "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps,
                      "config": {"workload": w.name, "schedule": sched},
                      "roofline": prefill_roofline(w, ms, peaks, sched),
                      "clocks": clk.summary()}), flush=True)


def prefill_roofline(w, ms, peaks, sched, traffic=None):
    """Roofline of one prefill call: the method's FLOPs (chunked contractions at tile
    shape) and algorithmic bytes over the call's device time."""
    flops = prefill_flops_per_token_head(w.dk, w.dv) * w.tokens * w.H_v
    tf = flops / (ms * 1e-3) / 1e12
    byt = prefill_bytes(w)
    return {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tf / peaks["bf16_tflops"], "traffic": traffic,
            "peak_src": f"{peaks['source']} bf16 burst", "flops": flops, "bytes": byt,
            "hbm_frac": byt / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "kernel": sched["kernel"], "launches": sched["launches"]}


def short_section(name, value, unit, ms, roof=None, **kw):
    d = {"w": name, "value": value, "unit": unit, "ms": ms}
    if roof is not None:
        d["frac"] = roof["frac"]
        d["achieved"] = roof["achieved"]
        d["bound"] = roof["bound"]
    d.update(kw)
    return d


def run_ours(args):
    if args.section == "qsa":
        return run_qsa_only(args)
    if args.section == "prefill":
        return run_prefill_only(args)
    rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import linear_attention_token_b200 as gdn
    gdn.lib()                                   # loud failure if libgdn.so is missing
    peaks = load_peaks()
    wp, wm, wv, wd = (inputs.get(i) for i in (PREFILL_W, MID_W, VARLEN_W, DECODE_W))
    stream = torch.cuda.Stream(device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    warm = max(args.warmup, 3)
    launches = 0

    barrier(world)
    with ClockSampler(local) as clk:
        x = inputs.prefill_inputs(wp, device=device)
        times, status, sched = time_prefill(gdn, x, wp, args.steps, warm, stream, flush)
        launches += args.steps * sched["launches"]
        del x
        torch.cuda.empty_cache()
        barrier(world)
        dec_passes = max(1, min(args.steps, 5))
        dtimes = time_decode(gdn, wd, dec_passes, max(1, min(args.warmup, 3)), stream, device)
        launches += dec_passes * wd.decode_steps
        barrier(world)
        sec_steps = max(3, min(args.steps, 10))
        xm = inputs.prefill_inputs(wm, device=device)
        mtimes_p, st_m, sched_m = time_prefill(gdn, xm, wm, sec_steps, warm, stream, flush)
        launches += sec_steps * sched_m["launches"]
        bw_steps = max(1, min(args.steps, 3))
        btimes = time_backward(gdn, xm, wm, bw_steps, 1, stream)
        launches += bw_steps
        del xm
        barrier(world)
        xv = inputs.prefill_inputs(wv, device=device)
        vtimes_p, st_v, sched_v = time_prefill(gdn, xv, wv, sec_steps, warm, stream, flush)
        launches += sec_steps * sched_v["launches"]
        del xv
        torch.cuda.empty_cache()
        barrier(world)
        vtimes, v_calls = time_decode_multi(gdn, wd, VERIFY_T, dec_passes, max(1, min(args.warmup, 3)),
                                            stream, device)
        launches += dec_passes * v_calls
        barrier(world)
        wq = qsa_workload(args)
        q_steps = max(3, min(args.steps, 20))
        qtimes, ctimes, q_blocks, q_tokens, mtimes = time_qsa(gdn, wq, q_steps, 3, stream, device)
        launches += 3 * len(qtimes) + 3 * len(mtimes) + len(ctimes)
        barrier(world)
    clocks = clk.summary()
    for st in (status, st_m, st_v):
        if st != 0:
            raise RuntimeError(f"device error after prefill: {gdn.gdn_status_string(st)}")

    ms_prefill = max_over_ranks(sum(times) / len(times), world)
    ms_decode_pass = max_over_ranks(sum(dtimes) / len(dtimes), world)
    e2e_steps = max(2, min(args.steps, 4))
    e2e_times, h2d, d2h = time_prefill_e2e(gdn, wp, e2e_steps, 1, stream, device)
    launches += e2e_steps * sched["launches"]
    ms_e2e = max_over_ranks(sum(e2e_times) / len(e2e_times), world)

    tok = wp.tokens
    pf_src = os.path.join(ROOT, "linear_attention_token_b200", "csrc", "prefill_chain.cu")
    roof = prefill_roofline(wp, ms_prefill, peaks, sched, profiled_traffic("prefill_long", pf_src))
    ms_dec_step = ms_decode_pass / wd.decode_steps
    dec_bytes = decode_bytes_per_step(wd)
    dec_gbs = dec_bytes / (ms_dec_step * 1e-3) / 1e9
    dec_src = os.path.join(ROOT, "linear_attention_token_b200", "csrc", "decode.cu")
    ms_m = max_over_ranks(sum(mtimes_p) / len(mtimes_p), world)
    ms_v = max_over_ranks(sum(vtimes_p) / len(vtimes_p), world)
    ms_verify_pass = max_over_ranks(sum(vtimes) / len(vtimes), world)
    ms_bw = max_over_ranks(sum(btimes) / len(btimes), world)
    ver_bytes = decode_multi_bytes_per_call(wd, VERIFY_T)
    ver_gbs = ver_bytes / (ms_verify_pass / v_calls * 1e-3) / 1e9
    qsa = qsa_section(gdn, peaks, wq, qtimes, ctimes, q_blocks, q_tokens, world, mtimes)
    rm = prefill_roofline(wm, ms_m, peaks, sched_m)
    rv = prefill_roofline(wv, ms_v, peaks, sched_v)

    line = {
        "metric": METRIC,
        "value": job_tokens_per_s(world, tok, ms_prefill),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": warm,
        "ms_per_step": ms_prefill,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; q,k ~ N(0,1) L2-normalised, v ~ N(0,1), g = -0.1 softplus(N(0,1)), "
                "beta = sigmoid(N(0,1)))",
        "config": prefill_config(wp, world, sched),
        "roofline": roof,
        "e2e": {"value": world * tok / (ms_e2e * 1e-3), "unit": "tokens/s", "ms": ms_e2e,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "decode": {
            "w": wd.name, "value": world * wd.decode_seqs / (ms_dec_step * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms_dec_step, "passes": dec_passes,
            "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                         "traffic": profiled_traffic("decode", dec_src), "bytes": dec_bytes}},
        "gpu_launches": launches,
        "clocks": clocks,
        "sections": {
            "mid": short_section(wm.name, world * wm.tokens / (ms_m * 1e-3), "tokens/s", ms_m, rm,
                                 kernel=sched_m["kernel"], seg=sched_m["segment_tokens"]),
            "varlen": short_section(wv.name, world * wv.tokens / (ms_v * 1e-3), "tokens/s", ms_v, rv,
                                    kernel=sched_v["kernel"], seg=sched_v["segment_tokens"]),
            "dec_multi": short_section(f"{wd.name} as {VERIFY_T}-token calls",
                                       world * wd.decode_seqs * wd.decode_steps / (ms_verify_pass * 1e-3),
                                       "tokens/s", ms_verify_pass / v_calls,
                                       {"frac": ver_gbs / peaks["hbm_gbs"], "achieved": ver_gbs, "bound": "hbm"}),
            "backward": short_section(wm.name, world * wm.tokens / (ms_bw * 1e-3), "tokens/s", ms_bw),
            "qsa": short_section(qsa["workload"], qsa["value"], "queries/s", qsa["ms_per_call"],
                                 qsa["roofline"],
                                 multi={"value": qsa["multi_query"]["value"],
                                        "ms": qsa["multi_query"]["ms_per_call"],
                                        "frac": qsa["multi_query"]["roofline"]["frac"]},
                                 compress={"value": qsa["compress"]["value"],
                                           "ms": qsa["compress"]["ms_per_call"],
                                           "frac": qsa["compress"]["roofline"]["frac"]}),
        },
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline_prefill(wp, max_tokens=CPU_PREFIX)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
        db = cpu_baseline_decode(wd)
        line["decode"]["cpu_baseline"] = {"value": db["value"], "unit": db["unit"], "cores": db["cores"]}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


CPU_PREFIX = 65536     # tokens of the long-context workload the oracle baseline runs


def prefill_config(wp, world, sched=None):
    d = {"workload": wp.name, "B": len(wp.seq_lens), "T": wp.seq_lens[0], "H_qk": wp.H_qk,
         "H_v": wp.H_v, "dk": wp.dk, "dv": wp.dv, "chunk": CHUNK, "state": "fp32",
         "parallelism": f"replicas x{world}" if world > 1 else "single",
         "l2": "inputs 4.3 GB > L2; a 256 MB buffer is also written between steps"}
    if sched is not None:
        d["schedule"] = f"{sched['kernel']}, segments of {sched['segment_tokens']} tokens" \
            if sched["segment_tokens"] else sched["kernel"]
    return d


def run_reference(args):
    """The oracle as it stands, on the host cores, on our arm's workload and metric: every
    step runs the sequential recurrence over a prefix of the long-context workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wp = inputs.get(PREFILL_W)
    prefix = 16384
    for _ in range(args.warmup):
        cpu_baseline_prefill(wp, max_tokens=1024)
    runs = [cpu_baseline_prefill(wp, max_tokens=prefix) for _ in range(args.steps)]
    secs = [r["seconds"] for r in runs]
    ntok = min(prefix, wp.tokens)
    ms = 1e3 * sum(secs) / len(secs)
    v = ntok / (ms * 1e-3)
    base = dict(runs[0])
    base.pop("seconds", None)
    base["value"] = v
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "device": "host cores (the oracle; no GPU work)",
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": prefill_config(wp, args.gpus),
        "cpu_baseline": base,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--section", choices=["all", "qsa", "prefill"], default="all",
                    help="qsa: time only the QSA indexer and compression; prefill: one prefill "
                         "workload alone (profiling aids)")
    ap.add_argument("--prefill-workload", type=int, choices=[1, 2, 3], default=PREFILL_W,
                    help="--section prefill: the workload (1 mid-size, 2 varlen, 3 long context)")
    ap.add_argument("--prefill-tokens", type=int, default=0,
                    help="--section prefill: keep only the first N tokens of each sequence")
    ap.add_argument("--segment-tokens", type=int, default=0,
                    help="--section prefill: schedule override (0 automatic, -1 one unit per "
                         "sequence, -2 cluster kernel, else a segment length)")
    ap.add_argument("--qsa-seqs", type=int, default=8,
                    help="sequences of the QSA workload (1,048,576 cached tokens each)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
