"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The layer does not shard (one KV-head group's state is one GPU's work), so several GPUs run
independent replicas: the only collectives are the barrier around the timed region and the
max over ranks of the device time.  These run here on gloo with two ranks.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    r, w = bench.dist_init("gloo")
    bench.barrier()
    got = bench.max_over_ranks(10.0 + 5.0 * rank)
    ref = bench.run_reference(type("A", (), dict(workload="mistral_128k", warmup=0, steps=0))(), r, w) \
        if rank == 1 else "rank0-skipped"
    bench.barrier()
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, r, w, got, ref))


def test_max_over_ranks_and_reference_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    assert all(x[2] == 2 for x in res)
    assert all(x[3] == 15.0 for x in res)  # the slowest rank's time
    assert res[1][4] is None  # rank 1 does no oracle work for the reference arm


def test_single_process_defaults():
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.max_over_ranks(3.5) == 3.5
