"""KV-head sharding of one InfLLM attention layer over the GPUs of a node (one process per GPU).

Every KV group of the layer is independent: its memory units, representative tokens, unit scores,
top-k selection and softmax involve only that KV head and the q heads that read it ("InfLLM Guide:
Training-Free Long-Context Memory Units", "Core Innovation 2": the lookup and the exact attention
are per head; q head h reads KV head h // (Hq / Hkv)).  So rank r of N holds KV heads
[r Hkv / N, (r + 1) Hkv / N) together with their q heads and runs the layer on that slice with no
exchange inside the layer; only the outputs are gathered, which in a model is the tensor-parallel
step that follows attention.  `gather_heads` does it with torch.distributed.all_gather (NCCL over
NVLink between GPUs of a node, gloo on CPU).

This module is host logic and argument marshalling only: each rank's slice runs through the same
C-ABI kernels as an unsharded layer (`ShardedLayer` wraps `InfLLMLayer`).
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class ShardPlan:
    """Which heads rank `rank` of `world` holds: KV heads [kv0, kv1), q heads [q0, q1)."""
    n_q_heads: int
    n_kv_heads: int
    world: int
    rank: int

    def __post_init__(self):
        if self.world < 1 or not 0 <= self.rank < self.world:
            raise ValueError(f"rank {self.rank} outside world of {self.world}")
        if self.n_q_heads % self.n_kv_heads:
            raise ValueError("n_q_heads must be a multiple of n_kv_heads")
        if self.n_kv_heads % self.world:
            raise ValueError(f"{self.n_kv_heads} KV heads do not split evenly over {self.world} ranks")

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def kv_per_rank(self) -> int:
        return self.n_kv_heads // self.world

    @property
    def kv0(self) -> int:
        return self.rank * self.kv_per_rank

    @property
    def kv1(self) -> int:
        return self.kv0 + self.kv_per_rank

    @property
    def q0(self) -> int:
        return self.kv0 * self.group

    @property
    def q1(self) -> int:
        return self.kv1 * self.group

    def local_config(self, cfg: dict) -> dict:
        """The layer configuration of this rank's slice (same shape, fewer heads)."""
        return dict(cfg, n_q_heads=self.q1 - self.q0, n_kv_heads=self.kv1 - self.kv0)

    def slice_q(self, q):
        """q [n, Hq, d] -> this rank's heads [n, Hq / N, d] (contiguous)."""
        return q[:, self.q0:self.q1].contiguous()

    def slice_kv(self, x):
        """k or v [n, Hkv, d] -> this rank's heads [n, Hkv / N, d] (contiguous)."""
        return x[:, self.kv0:self.kv1].contiguous()


def gather_heads(local_out, plan: ShardPlan, group=None):
    """All ranks' outputs [n, Hq / N, d] -> the full output [n, Hq, d] on every rank (rank r's heads at
    [r Hq / N, (r + 1) Hq / N), which is the unsharded order)."""
    import torch
    import torch.distributed as dist
    if plan.world == 1:
        return local_out
    parts = [torch.empty_like(local_out) for _ in range(plan.world)]
    dist.all_gather(parts, local_out.contiguous(), group=group)
    return torch.cat(parts, dim=1)


class ShardedLayer:
    """One rank's share of a layer.  `make_layer(local_cfg)` builds the rank's layer (by default an
    InfLLMLayer on the current device); inputs are full-head tensors, outputs are gathered unless
    `gather=False`."""

    def __init__(self, cfg: dict, plan: ShardPlan, make_layer=None, group=None, **layer_kw):
        self.plan = plan
        self.group = group
        local = plan.local_config(cfg)
        if make_layer is None:
            from . import InfLLMLayer
            self.layer = InfLLMLayer(**local, **layer_kw)
        else:
            self.layer = make_layer(local)

    def _out(self, local_out, gather):
        return gather_heads(local_out, self.plan, self.group) if gather else local_out

    def prefill(self, q, k, v, chunk, gather=True):
        p = self.plan
        return self._out(self.layer.prefill(p.slice_q(q), p.slice_kv(k), p.slice_kv(v), chunk), gather)

    def append_chunk(self, q, k, v):
        p = self.plan
        self.layer.append_chunk(p.slice_q(q), p.slice_kv(k), p.slice_kv(v))

    def attend_chunk(self, q, gather=True):
        return self._out(self.layer.attend_chunk(self.plan.slice_q(q)), gather)

    def decode_step(self, q, k, v, gather=True):
        p = self.plan
        return self._out(self.layer.decode_step(p.slice_q(q), p.slice_kv(k), p.slice_kv(v)), gather)

    def close(self):
        close = getattr(self.layer, "close", None)
        if close:
            close()
