"""The N > 1 path of bench.py, on CPU with two gloo ranks: the layer has no exchange
between GPUs, so N GPUs run N replicas and only the barrier, the max-over-ranks timing
and the whole-job throughput cross between ranks.  Also: a rank that leaves before the
barrier makes the others' next collective fail with an error within the process
group's timeout, instead of hanging."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        r, w, _ = bench.dist_init(backend="gloo", timeout_s=5.0)
        assert (r, w) == (rank, world)
        if mode == "ok":
            bench.barrier(w)
            ms = bench.max_over_ranks(10.0 + 5.0 * rank, w)      # rank times 10 and 15 ms
            value = bench.job_tokens_per_s(w, 8192, ms)
            bench.barrier(w)
            q.put((rank, "ok", ms, value))
        else:                                                    # rank 1 leaves early
            if rank == 1:
                q.put((rank, "left", None, None))
                return
            try:
                bench.barrier(w)
                q.put((rank, "no error", None, None))
            except Exception as e:                               # noqa: BLE001
                q.put((rank, "error", type(e).__name__, None))
    finally:
        if dist.is_initialized():
            try:
                dist.destroy_process_group()
            except Exception:                                    # noqa: BLE001
                pass


def _run(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    return sorted(out)


def test_two_replicas_time_is_the_slowest_and_value_counts_both():
    out = _run("ok")
    assert [o[1] for o in out] == ["ok", "ok"]
    for _, _, ms, value in out:
        assert ms == 15.0                                  # the max over ranks, on every rank
        assert value == pytest.approx(2 * 8192 / 15e-3)    # both replicas' tokens


def test_a_rank_that_leaves_makes_the_next_collective_fail():
    out = _run("leave")
    assert out[1][1] == "left"
    assert out[0][1] == "error"                            # not a hang: the timeout fired
