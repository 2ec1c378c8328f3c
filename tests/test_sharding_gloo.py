"""KV-head sharding of one layer over several ranks, on CPU (gloo, world size 2 and 4).

The per-rank compute here is the fp64 oracle on the rank's head slice (the CUDA kernels need a GPU;
a rank's slice runs through them unchanged on a GPU node).  What is checked is the sharding itself:
the plan covers every KV head once with its own q heads, and running the slices on separate ranks
and gathering the heads gives exactly the unsharded layer's outputs, selections included -- the KV
groups share nothing inside the layer.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from block_memory_sparse_b200.sharding import ShardPlan


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


CFG = dict(n_q_heads=8, n_kv_heads=4, head_dim=16, n_sink=3, window=40, unit_size=8, n_reps=2, top_k=3,
           rope_base=1e4, dtype="f32")
T, CHUNK = 230, 37


def _inputs():
    r = np.random.default_rng(7)
    q = r.standard_normal((T, CFG["n_q_heads"], CFG["head_dim"]))
    k = r.standard_normal((T, CFG["n_kv_heads"], CFG["head_dim"])) + 2.0 * r.standard_normal((1, CFG["n_kv_heads"], 1))
    v = r.standard_normal((T, CFG["n_kv_heads"], CFG["head_dim"]))
    return q, k, v


class OracleChunks:
    """The oracle behind the layer interface ShardedLayer drives (prefill of a whole prompt)."""

    def __init__(self, cfg):
        from oracle import infllm_oracle as O
        self.layer = O.OracleLayer(cfg, rep_method="linear")
        self.sels = []

    def prefill(self, q, k, v, chunk):
        out = []
        for c0 in range(0, q.shape[0], chunk):
            n = min(chunk, q.shape[0] - c0)
            self.layer.append_chunk(q[c0:c0 + n].numpy(), k[c0:c0 + n].numpy(), v[c0:c0 + n].numpy())
            out.append(self.layer.attend_chunk())
            self.sels.append(self.layer.last["sel"])
        return torch.from_numpy(np.concatenate(out))


def _worker(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from block_memory_sparse_b200.sharding import ShardedLayer
    dist.init_process_group("gloo", rank=rank, world_size=world)
    plan = ShardPlan(CFG["n_q_heads"], CFG["n_kv_heads"], world, rank)
    q, k, v = (torch.from_numpy(a) for a in _inputs())
    layer = ShardedLayer(CFG, plan, make_layer=OracleChunks)
    out = layer.prefill(q, k, v, CHUNK)
    sels = layer.layer.sels
    dist.barrier()
    dist.destroy_process_group()
    q_out.put((rank, out.numpy(), sels))


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_prefill_equals_unsharded(world):
    from oracle import infllm_oracle as O
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = OracleChunks(CFG)
    q, k, v = (torch.from_numpy(a) for a in _inputs())
    ref = full.prefill(q, k, v, CHUNK).numpy()
    assert O.n_mem(T - (T % CHUNK), CFG["n_sink"], CFG["window"], CFG["unit_size"]) > CFG["top_k"]
    kvr = CFG["n_kv_heads"] // world
    for rank, out, sels in res:
        np.testing.assert_array_equal(out, ref)  # every rank holds the gathered, unsharded output
        for ci, sel in enumerate(sels):  # each rank's selections are the unsharded ones of its KV heads
            assert sel == full.sels[ci][rank * kvr:(rank + 1) * kvr]


@pytest.mark.parametrize("hq,hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (8, 8, 4), (16, 2, 2)])
def test_plan_covers_every_head_once(hq, hkv, world):
    kv_seen, q_seen = [], []
    for r in range(world):
        p = ShardPlan(hq, hkv, world, r)
        kv_seen += list(range(p.kv0, p.kv1))
        q_seen += list(range(p.q0, p.q1))
        for h in range(p.q0, p.q1):  # a q head travels with the KV head it reads
            assert p.kv0 <= h // (hq // hkv) < p.kv1
        lc = p.local_config(dict(n_q_heads=hq, n_kv_heads=hkv, head_dim=128))
        assert lc["n_q_heads"] // lc["n_kv_heads"] == hq // hkv
    assert kv_seen == list(range(hkv)) and q_seen == list(range(hq))


def test_plan_refuses_uneven_splits():
    with pytest.raises(ValueError):
        ShardPlan(32, 8, 3, 0)
    with pytest.raises(ValueError):
        ShardPlan(32, 8, 2, 2)
