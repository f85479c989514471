"""Expert parallelism over several GPUs (one process per GPU, torch.distributed over NCCL).

The routed experts of every layer are the shard: rank r of G holds the blobs of the experts
e with e % G == r (round-robin, so each rank gets an equal share of any popularity ranking),
in its own pool at slot e // G; the router, the shared-expert gate and the shared expert are
replicated.  A layer on T tokens is then

    every rank        routes the same tokens (same inputs, same deterministic kernel: the
                      same top-k everywhere)
    every rank        moe_layer_forward_partial: the fp32 partial output over its own
                      selected experts (the others' slot-table entries say "held by another
                      rank"); rank 0 adds the shared expert
    all ranks         one sum all-reduce of the [T, H] fp32 partials (8 KB per token)
    every rank        moe_combine_partials: out = bf16(sum + residual)

This module holds the partition and the plumbing only; every arithmetic step of the layer
runs in the library's kernels, and the collective is NCCL's (torch.distributed).
"""
from __future__ import annotations

from typing import Optional

import torch

SLOT_REMOTE = -3  # slot-table entry of an expert held by another rank


def owner(expert: int, world: int) -> int:
    """Rank that holds `expert`."""
    return expert % world


def local_experts(n_experts: int, rank: int, world: int):
    """The experts rank `rank` holds, in slot order (slot i holds the i-th of them)."""
    return list(range(rank, n_experts, world))


def local_slot_table(n_experts: int, rank: int, world: int, device=None) -> torch.Tensor:
    """int32 [E]: slot e // world for this rank's experts, SLOT_REMOTE for the others."""
    e = torch.arange(n_experts, dtype=torch.int32)
    t = torch.where(e % world == rank, e // world, torch.full_like(e, SLOT_REMOTE))
    return t.to(device) if device is not None else t


def shard_pool(full_pool: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """This rank's pool [ceil(E / world) or fewer, stride] from a full pool [E, stride]."""
    return full_pool[rank::world].contiguous()


class EPLayer:
    """One routed-MoE layer of an expert-parallel stack on this rank.

    pool / slot_table are this rank's shard (see shard_pool / local_slot_table); the rest
    is replicated.  forward() runs the partial, the all-reduce and the combine on `stream`.
    """

    def __init__(self, shape, w_router, router_bias, pool, slot_table, shared_blob, w_shared_gate, rank: int,
                 world: int, T: int, device, group=None):
        from . import abi
        self.abi = abi
        self.shape, self.T, self.rank, self.world, self.group = shape, T, rank, world, group
        self.w_router, self.router_bias = w_router, router_bias
        self.pool, self.slot_table = pool, slot_table
        self.shared, self.w_sg = shared_blob, w_shared_gate
        self.partial = torch.zeros(T, shape.hidden, dtype=torch.float32, device=device)
        self.ws = torch.zeros(abi.moe_workspace_size(shape, T), dtype=torch.uint8, device=device)

    def forward(self, x, residual, out, topk_idx_out=None, topk_w_out=None, stream=None):
        import torch.distributed as dist
        a = self.abi
        a.moe_layer_forward_partial(self.shape, x, self.T, self.w_router, self.router_bias, None, None, self.pool,
                                    self.slot_table, self.pool.shape[0], self.shared, self.w_sg,
                                    1 if self.rank == 0 else 0, self.partial, topk_idx_out, topk_w_out, self.ws,
                                    stream)
        if self.world > 1:
            dist.all_reduce(self.partial, op=dist.ReduceOp.SUM, group=self.group)
        a.moe_combine_partials([self.partial], self.T, self.shape.hidden, residual, out, stream)
