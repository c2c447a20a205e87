"""Replica plumbing of bench.py on the host: two ranks without a GPU (gloo) set
up the process group the way bench.py does, agree on the slowest rank's step
time, and report the whole job's throughput as every rank's units over that
time.  The layer itself does not shard: each rank runs an independent replica."""
import os
import queue
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    w, r, _ = bench.dist_setup(world, timeout_s=60)
    try:
        bench.barrier(w)
        step_ms = 2.0 + r                       # the last rank is the slowest
        slowest = bench.max_over_ranks(step_ms, w)
        out.put((r, w, torch.distributed.get_backend(), slowest, bench.replica_throughput(1000, w, slowest)))
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_rank():
    if torch.cuda.is_available():
        pytest.skip("host-side test: with a GPU the plumbing uses NCCL, one GPU per rank")
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = []
    try:
        for _ in range(2):
            got.append(out.get(timeout=120))
    except queue.Empty:
        pass
    for p in procs:
        p.join(60)
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    assert sorted(g[0] for g in got) == [0, 1]
    for rank, world, backend, slowest, rate in got:
        assert world == 2 and backend == "gloo"
        assert slowest == 3.0
        assert rate == pytest.approx(2 * 1000 / 3e-3)
