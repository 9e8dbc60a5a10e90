"""Head sharding of one attention layer across ranks: tensor parallelism over heads, no collective.

The FlashMLA-ETAP summary ("Planteamiento del Problema", item 1) describes serving a 128-head
model on one 8-GPU instance with 16 heads per GPU: attention heads are independent, so each GPU
computes its own heads against the K/V they read and the outputs stay sharded for the next
(head-parallel) projection. This module holds the host-side arithmetic of that split; every rank
then calls the ordinary entry points on its shard.

Rules (GQA: query head h reads kv head h // G, G = Hq / Hkv):
  * Hq must divide evenly over the ranks: rank r owns query heads [r * Hq/N, (r + 1) * Hq/N);
  * if Hq/N is a multiple of G each rank owns whole groups and their kv heads;
  * if G is a multiple of Hq/N a group spans several ranks and each of them holds a copy of that
    one kv head (MLA: one latent head shared by all 128 query heads, replicated on every GPU);
  * any other split would cut a group unevenly and is rejected.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class HeadShard:
    rank: int
    world: int
    q_heads: tuple  # [h0, h1)
    kv_heads: tuple  # [k0, k1)

    @property
    def Hq(self) -> int:
        return self.q_heads[1] - self.q_heads[0]

    @property
    def Hkv(self) -> int:
        return self.kv_heads[1] - self.kv_heads[0]


def head_shard(Hq: int, Hkv: int, world: int, rank: int) -> HeadShard:
    """The query and kv heads rank `rank` of `world` owns (see the module notes for the rules)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if Hq < 1 or Hkv < 1 or Hq % Hkv:
        raise ValueError(f"Hq={Hq} must be a positive multiple of Hkv={Hkv}")
    if Hq % world:
        raise ValueError(f"{Hq} query heads do not split evenly over {world} ranks")
    G = Hq // Hkv
    per = Hq // world
    h0, h1 = rank * per, (rank + 1) * per
    if per % G == 0:
        kv = (h0 // G, h1 // G)
    elif G % per == 0:
        kv = (h0 // G, h0 // G + 1)
    else:
        raise ValueError(f"{per} query heads per rank would split groups of {G} unevenly")
    return HeadShard(rank, world, (h0, h1), kv)


def shard_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shard: HeadShard):
    """Contiguous per-rank copies of q [B, Hq, Lq, d], k [B, Hkv, Lk, d] and v (v may be k itself:
    latent KV, then the returned v is the returned k)."""
    h0, h1 = shard.q_heads
    k0, k1 = shard.kv_heads
    qs = q[:, h0:h1].contiguous()
    ks = k[:, k0:k1].contiguous()
    vs = ks if v is k else v[:, k0:k1].contiguous()
    return qs, ks, vs


def gather_heads(parts) -> torch.Tensor:
    """Reassemble per-rank outputs [B, Hq/N, ...] in rank order (host-side, for checking)."""
    return torch.cat(list(parts), dim=1)
