"""The multi-GPU path of bench.py is replicas only (no exchange step on the data path): every
rank runs its own stream and the job's throughput is all ranks' work over the slowest rank's
device time.  These tests run that host logic as 2 gloo ranks on CPU, including a rank that
dies before the exchange (the survivor must fail with an error, not hang)."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        dist = bench._init_dist(world, backend="gloo", timeout_s=10)
        if mode == "die" and rank == 1:
            os._exit(3)                       # leaves before the exchange, between steps
        elapsed = [0.50, 0.75][rank]          # device-timed seconds of this rank
        t_max, tflops = bench.aggregate(dist, elapsed, 2.0e12, torch.device("cpu"))
        q.put((rank, "ok", t_max, tflops))
        dist.destroy_process_group()
    except Exception as e:                     # reported to the parent, never swallowed
        q.put((rank, "error", type(e).__name__, str(e)[:200]))


def _run(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    out = []
    while not q.empty():
        out.append(q.get())
    return sorted(out), [p.exitcode for p in procs], alive


def test_replicas_max_time_and_summed_work():
    out, codes, alive = _run("ok")
    assert not alive and codes == [0, 0]
    for rank, status, t_max, tflops in out:
        assert status == "ok"
        assert t_max == pytest.approx(0.75)            # the slowest rank's time
        assert tflops == pytest.approx(2 * 2.0 / 0.75)  # both ranks' work over it


def test_dead_rank_fails_the_survivor_quickly():
    out, codes, alive = _run("die")
    assert not alive, "a rank hung instead of failing"
    assert codes[1] == 3
    assert [o[:2] for o in out] == [(0, "error")]
