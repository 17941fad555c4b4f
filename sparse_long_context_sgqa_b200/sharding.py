"""KV-group sharding of the hot path over up to four GPUs (one process per GPU).

Page "Step-5-Preview: Sparse Reads Are Not a Compressed KV Cache", section
"Cache capacity: 4,104 reads do not mean 4,104 stored tokens": the four KV
groups are independent -- each has its own K/V, its own 16 query heads, its
own indexer heads and its own selection -- and only the merged search store
(built from the proxy keys, which every group shares) is common.  Rank r of
W (W divides G) therefore holds groups [r G / W, (r + 1) G / W): its slice of
the K/V cache, of the query heads and of the indexer queries and weights.  It
merges the shared store itself (cheap next to a cross-GPU copy) and runs the
whole path for its groups with ``num_kv_groups = G / W``.  The path has no
exchange step; the only collective is the optional all-gather of the output
heads for a replicated output projection (NCCL over NVLink through
``torch.distributed``).

Layouts follow include/sgqa.h: heads of group g are g*Hg .. g*Hg + Hg - 1, so
a rank's heads and groups are contiguous slices of the full tensors.
"""
from __future__ import annotations

import dataclasses

import torch


def group_range(num_groups: int, world: int, rank: int):
    """KV groups [g0, g1) that `rank` of `world` holds."""
    if world < 1 or num_groups % world != 0:
        raise ValueError(f"{world} ranks cannot split {num_groups} KV groups evenly")
    per = num_groups // world
    return rank * per, (rank + 1) * per


def shard_queries(q, idx_q, idx_w, num_groups: int, heads_per_group: int, world: int, rank: int):
    """This rank's slices of the query-side tensors (contiguous copies):
    q [S, N, G*Hg, D] -> heads of its groups; idx_q [S, N, G, H, Di] and
    idx_w [S, N, G, H] -> its groups."""
    g0, g1 = group_range(num_groups, world, rank)
    return (q[:, :, g0 * heads_per_group:g1 * heads_per_group].contiguous(),
            idx_q[:, :, g0:g1].contiguous(), idx_w[:, :, g0:g1].contiguous())


def shard_kv(k, v, num_groups: int, world: int, rank: int):
    """This rank's groups of the K/V caches [S, cap, G, D] (contiguous copies)."""
    g0, g1 = group_range(num_groups, world, rank)
    return k[:, :, g0:g1].contiguous(), v[:, :, g0:g1].contiguous()


def gather_heads(local_out: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather every rank's output heads [S, N, Gl*Hg, D] into the full
    [S, N, W*Gl*Hg, D], rank r's heads at their global position."""
    if world == 1:
        return local_out
    dist = torch.distributed
    S, N, Hl, D = local_out.shape
    flat = torch.empty((world * S, N, Hl, D), dtype=local_out.dtype, device=local_out.device)
    dist.all_gather_into_tensor(flat, local_out.contiguous(), group=group)  # rank r's heads at rows r*S ..
    return flat.view(world, S, N, Hl, D).permute(1, 2, 0, 3, 4).reshape(S, N, world * Hl, D)


class GroupShardedSGQA:
    """One rank of a KV-group-sharded Sparse GQA layer.

    ``model`` is a SparseGQA-like object built with this rank's group count
    (``local_params``) whose ``forward(q_pos0, q, idx_q, idx_w, sel, sel_count,
    out, ...)`` runs the path on this rank's slices; its caches hold this
    rank's K/V groups and the full proxy keys and logits.
    """

    def __init__(self, params, world: int, rank: int, make_model, group=None):
        self.world, self.rank, self.group = world, rank, group
        self.full = params
        self.g0, self.g1 = group_range(params.num_kv_groups, world, rank)
        self.local_params = dataclasses.replace(params, num_kv_groups=self.g1 - self.g0)
        self.model = make_model(self.local_params)

    def load_cache(self, kp, c, k, v):
        """Fill this rank's caches from full-cache tensors (positions [0, L))."""
        L = kp.shape[1]
        kl, vl = shard_kv(k, v, self.full.num_kv_groups, self.world, self.rank)
        self.model.kp[:, :L].copy_(kp)
        self.model.c[:, :L].copy_(c)
        self.model.k[:, :L].copy_(kl)
        self.model.v[:, :L].copy_(vl)

    def forward(self, q_pos0, q, idx_q, idx_w, gather: bool = True, **kw):
        """The path for this rank's groups on full query tensors; returns the
        full output (all ranks' heads, gathered) or this rank's heads only."""
        Hg = self.full.heads_per_group
        ql, iql, iwl = shard_queries(q, idx_q, idx_w, self.full.num_kv_groups, Hg, self.world, self.rank)
        S, N = q.shape[0], q.shape[1]
        Gl = self.g1 - self.g0
        sel = torch.empty((S, N, Gl, self.full.topk), dtype=torch.int32, device=q.device)
        cnt = torch.empty((S, N, Gl), dtype=torch.int32, device=q.device)
        out = torch.empty((S, N, Gl * Hg, q.shape[-1]), dtype=q.dtype, device=q.device)
        self.model.forward(q_pos0, ql, iql, iwl, sel, cnt, out, **kw)
        self.last_sel, self.last_cnt = sel, cnt
        return gather_heads(out, self.world, self.group) if gather else out
