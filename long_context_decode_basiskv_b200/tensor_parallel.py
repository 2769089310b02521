"""Head-sharded (tensor-parallel) decode step: each rank holds a slice of the KV groups.

The BasisKV pages deploy the method under tensor parallelism, with the
attention heads partitioned across GPUs (BasisKV abstract; kongchang.com
explainer, section "分布式推理中被忽视的通信成本").  With the Value latent
fused into the output projection (G_h = B_g W_O,h), rank i owning the KV
groups [i Hkv/N, (i+1) Hkv/N) and their query heads computes every step of
the decode path for its heads alone (append, route, attention, and the
partial out-projection y_i = sum over its heads of o_h G_h) with the ordinary
single-GPU calls, and the layer output is y = sum_i y_i: one all-reduce of
B x hidden fp32 values per step.

``shard_case`` slices a seeded case by heads (no arithmetic: the factors,
W_O rows, queries and token rows of the rank's heads), so every rank builds
the same full case from the same seed and keeps its slice.  ``reduce_y``
is the exchange step.
"""
from __future__ import annotations

import dataclasses

import torch

from .workloads import Case


def head_range(num_kv_heads: int, rank: int, world: int):
    """KV groups [g0, g1) of `rank` out of `world` (equal contiguous slices)."""
    if world < 1 or num_kv_heads % world != 0:
        raise ValueError(f"{num_kv_heads} KV heads do not split over {world} ranks")
    per = num_kv_heads // world
    return rank * per, (rank + 1) * per


def shard_case(case: Case, rank: int, world: int) -> Case:
    """The slice of `case` that rank `rank` of `world` computes: its KV groups, their
    G query heads each, the factors of those groups and the W_O rows of those heads."""
    wl = case.wl
    g0, g1 = head_range(wl.num_kv_heads, rank, world)
    G = wl.num_q_heads // wl.num_kv_heads
    h0, h1 = g0 * G, g1 * G
    d = wl.head_dim
    swl = dataclasses.replace(wl, num_q_heads=h1 - h0, num_kv_heads=g1 - g0,
                              name=f"{wl.name}_tp{rank}of{world}")
    return dataclasses.replace(
        case, wl=swl,
        q=case.q[:, h0:h1].contiguous(),
        keys=[k[:, g0:g1].contiguous() for k in case.keys],
        values=[v[:, g0:g1].contiguous() for v in case.values],
        A=case.A[g0:g1].contiguous(), Bf=case.Bf[g0:g1].contiguous(),
        P=case.P[g0:g1].contiguous(), E=case.E[g0:g1].contiguous(),
        W_O=case.W_O[h0 * d:h1 * d].contiguous(),
        info=dict(case.info, tp_rank=rank, tp_world=world, kv_heads=(g0, g1), q_heads=(h0, h1)))


def reduce_y(y: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (the step's only exchange)."""
    if world > 1:
        torch.distributed.all_reduce(y, op=torch.distributed.ReduceOp.SUM, group=group)
    return y
