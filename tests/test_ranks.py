"""Multi-rank host logic of bench.py on CPU (gloo backend, world size 2).

The path shards by (batch, KV group) with no exchange step: every rank runs
its own independent problem, and the process group carries only the barrier
and the timing reduction (slowest rank's step, units summed over ranks).
These tests run that logic as two real processes, and check that a rank which
leaves without joining the collective ends the other rank's collective with
an error (short process-group timeout) instead of a hang.
"""
from __future__ import annotations

import importlib.util
import os
import socket
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, mode: str, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    try:
        bench = _bench()
        import bsa_workloads as W
        dist = bench.init_ranks(world, backend="gloo", timeout_s=5.0 if mode == "die" else 60.0)
        w = bench.rank_workload(W.get("prefill_gqa_bf16"), rank)
        if mode == "die" and rank == 1:
            os._exit(0)   # leaves before the collective, between steps
        t, u = bench.reduce_over_ranks(dist, 10.0 + rank, 100.0 * (rank + 1))
        q.put((rank, w.seed, t, u, None))
        bench.close_ranks(dist)
    except Exception as e:   # reported to the parent, which asserts on it
        q.put((rank, None, None, None, type(e).__name__))


def _run(mode: str, timeout: float = 120.0):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = []
    try:
        want = 2 if mode == "ok" else 1
        for _ in range(want):
            out.append(q.get(timeout=timeout))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
                p.join(timeout=10)
    return sorted(out, key=lambda r: r[0])


def test_two_ranks_reduce_timing_and_sum_units():
    res = _run("ok")
    assert [r[4] for r in res] == [None, None], res
    for rank, seed, t, u, _ in res:
        assert t == 11.0          # the slowest rank's step time
        assert u == 300.0         # 100 + 200 units
    seeds = {r[1] for r in res}
    assert len(seeds) == 2        # each rank its own independent problem


def test_rank_that_leaves_ends_the_other_ranks_collective():
    res = _run("die")
    assert len(res) == 1 and res[0][0] == 0
    assert res[0][4] is not None, "rank 0's collective should fail once rank 1 has left"


def test_single_rank_needs_no_process_group():
    bench = _bench()
    assert bench.init_ranks(1) is None
    assert bench.reduce_over_ranks(None, 2.5, 7.0) == (2.5, 7.0)
    bench.close_ranks(None)
