"""Tensor parallelism by KV head for the sparse decode step (host-side partitioning only).

Every (request, KV head) unit of the method is independent: its centroids, its group mean,
its scores, its top-k and its attention read only that KV head's pages and that head's G
query heads.  So N GPUs can each hold Hkv/N of the KV heads of every page -- K/V pool
[P, 16, Hkv/N, D], centroid cache [P, Hkv/N, D] -- together with the matching Hq/N query
heads, and run the whole step on their own with no exchange inside it; rank r's outputs are
the query heads [r Hq/N, (r+1) Hq/N) of the full result.  This is the tensor-parallel layout
the Vortex article reports on four B200s ("Speedups that scale to 229B parameters", TP=4);
the model's output projection that follows attention (and its all-reduce) is outside this
path.  The MLA latent form has one KV head and does not split this way: it is sharded by
request (data parallel) instead.

The functions here only compute head ranges and slice tensors; every step of the method runs
in the library's kernels on each rank.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class HeadShard:
    """The heads rank `rank` of `world` owns."""
    rank: int
    world: int
    kv0: int  # KV heads [kv0, kv1)
    kv1: int
    q0: int   # query heads [q0, q1)
    q1: int

    @property
    def num_kv_heads(self) -> int:
        return self.kv1 - self.kv0

    @property
    def num_q_heads(self) -> int:
        return self.q1 - self.q0


def kv_head_shard(num_q_heads: int, num_kv_heads: int, world: int, rank: int) -> HeadShard:
    """Contiguous, equal KV-head ranges; query head hq goes with KV head hq // G."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if num_kv_heads % world != 0:
        raise ValueError(f"{num_kv_heads} KV heads do not split evenly over {world} ranks "
                         "(the MLA latent form, with one KV head, shards by request instead)")
    if num_q_heads % num_kv_heads != 0:
        raise ValueError(f"{num_q_heads} query heads are not a multiple of {num_kv_heads}")
    G = num_q_heads // num_kv_heads
    per = num_kv_heads // world
    kv0 = rank * per
    return HeadShard(rank, world, kv0, kv0 + per, kv0 * G, (kv0 + per) * G)


def shard_pool(pool: torch.Tensor, s: HeadShard) -> torch.Tensor:
    """The shard's KV heads of a [P, 16, Hkv, D] pool: a strided view (the library takes any
    page / token / head strides), as a rank's own pool would hold them."""
    return pool[:, :, s.kv0:s.kv1]


def shard_queries(q: torch.Tensor, s: HeadShard) -> torch.Tensor:
    """The shard's query heads of q [B, Hq, D], contiguous (the library's layout for q)."""
    return q[:, s.q0:s.q1].contiguous()


def shard_centroids(centroids: torch.Tensor, s: HeadShard) -> torch.Tensor:
    """The shard's rows of a [P, Hkv, D] centroid cache, contiguous.  A rank that holds only
    its own heads builds this itself with vt_build_centroids on its pool shard."""
    return centroids[:, s.kv0:s.kv1].contiguous()


def gather_heads(parts: list, dim: int = 1) -> torch.Tensor:
    """Rank-ordered per-shard outputs (out [B, Hq/N, Dv], lse [B, Hq/N], sel [B, Hkv/N, k],
    n_sel [B, Hkv/N]) put back together along the head dimension."""
    return torch.cat(parts, dim=dim)
