"""Group sharding of one MSA layer over several GPUs.

Every step of the layer is independent per KV group: each group has its own
index query and its own top-k (lumi-systems AI news on MSA, on one top-k subset
per GQA group), the selection is shared only by the query heads of that group
(yhxrc.cn article on the MSA figure, section 第二步), and the one input that
all groups read, the index keys k_idx, is shared and read-only (same article,
section 第一步).  So world_size ranks can each own G / world_size consecutive
groups -- their K/V cache, the r query heads of each, their index queries --
plus a replica of k_idx, and run the unchanged single-GPU layer on that shard.
Nothing is exchanged inside the layer; rank i produces the output heads
[i*H/n, (i+1)*H/n).  A tensor-parallel projection after the layer would
gather or reduce those heads over NCCL.

Host-side partitioning only: the shard is an ordinary, smaller shape for the
C ABI (H/n query heads, G/n groups), and the compute runs in libmsa.
"""
from __future__ import annotations

from dataclasses import dataclass

from .msa import Shape, forward


@dataclass(frozen=True)
class GroupShard:
    rank: int
    world: int
    shape: Shape          # the shard's own shape: H/n query heads, G/n groups
    heads: tuple          # [h0, h1) of the full layer's query heads
    groups: tuple         # [g0, g1) of the full layer's KV groups


def group_shard(shape: Shape, rank: int, world: int) -> GroupShard:
    """Rank ``rank`` of ``world``'s share of ``shape``'s KV groups."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    G, H = shape.n_kv_heads, shape.n_q_heads
    if G % world:
        raise ValueError(f"{G} KV groups do not split over {world} ranks")
    gs = G // world
    r = H // G
    sub = Shape(*[getattr(shape, n) for n, _ in Shape._fields_])
    sub.n_kv_heads = gs
    sub.n_q_heads = gs * r
    g0 = rank * gs
    return GroupShard(rank, world, sub, (g0 * r, (g0 + gs) * r), (g0, g0 + gs))


def shard_inputs(sh: GroupShard, q, k, v, q_idx, k_idx):
    """The shard's inputs, contiguous, from full-layer tensors
    q [B, T, H, d], k / v [B, G, N, d], q_idx [B, T, G, d_i], k_idx [B, N, d_i].
    k_idx is replicated (returned as is)."""
    h0, h1 = sh.heads
    g0, g1 = sh.groups
    return (q[:, :, h0:h1].contiguous(), k[:, g0:g1].contiguous(), v[:, g0:g1].contiguous(),
            q_idx[:, :, g0:g1].contiguous(), k_idx)


def forward_group_shard(sh: GroupShard, q, k, v, q_idx, k_idx, **kw):
    """msa_forward on this rank's shard (inputs already sharded, see
    ``shard_inputs``).  Returns (o, lse, sel) for the shard's heads / groups."""
    return forward(sh.shape, q, k, v, q_idx, k_idx, **kw)
