"""Context-parallel decode of sequences whose keys are split over ranks.

One process per GPU; rank i holds the keys (index keys and latent rows) of
positions [offset_i, offset_i + len_i) of every sequence, the ranges in rank
order.  The step on each rank:

  1. indexer scores and exact top-k over its own keys      (its kernels)
  2. kept positions -> (score, global index) candidates     (dsa_cp_candidates)
  3. all-gather the candidates                              (NCCL)
  4. exact global top-k of the candidates, and this rank's
     share of it as local positions                         (dsa_cp_select)
  5. sparse MLA over its own kept rows                      (dsa_sparse_mla_decode)
  6. all-gather (out, lse)                                  (NCCL)
  7. log-sum-exp merge                                      (dsa_cp_merge)

Every rank ends with the same global indices and outputs, equal to the
one-device step over the whole sequence ("GLM on an A100, in Vx", "The model":
contexts of up to 1,048,576 tokens, 2,048 kept per query).  Only the two
all-gathers cross GPUs: 8 bytes per candidate and (4 R + 4) bytes per head.

`ops` carries the per-rank steps, the library's CUDA entry points by default;
the steps are passed in so that the exchange logic can be exercised by CPU
tests with stand-ins.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Callable


@dataclass
class RankShard:
    """This rank's part of the sequences: its key range and cache view."""
    offsets: Any          # [n_q] int32, global position of the first local key
    lens: Any             # [n_q] int32, local keys
    local: dict           # whatever the ops need for the local steps


@dataclass
class CpOps:
    local_topk: Callable          # (shard, k) -> (scores [n_q, ld], idx_local [n_q, k])
    candidates: Callable          # (scores, idx_local, offsets) -> (cand_s, cand_i) [n_q, k]
    select: Callable              # (all_s, all_i, offsets, lens) -> (gidx, own_idx) [n_q, k]
    attend: Callable              # (shard, own_idx) -> (out [n_q, H, dv], lse [n_q, H])
    merge: Callable               # (outs [R, ...], lses [R, ...]) -> (out, lse)


def all_gather_stacked(x, group, dist):
    """[R, *x.shape] of every rank's x, in rank order (every rank calls this)."""
    import torch
    world = dist.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def cp_decode_step(shard: RankShard, k: int, ops: CpOps, group=None, dist=None):
    """One context-parallel decode step; returns (gidx, out, lse), the same on
    every rank.  Every rank must call it, in the same order."""
    if dist is None:
        import torch.distributed as dist
    scores, idx_local = ops.local_topk(shard, k)
    cand_s, cand_i = ops.candidates(scores, idx_local, shard.offsets)
    all_s = all_gather_stacked(cand_s, group, dist)
    all_i = all_gather_stacked(cand_i, group, dist)
    gidx, own = ops.select(all_s, all_i, shard.offsets, shard.lens)
    out_r, lse_r = ops.attend(shard, own)
    outs = all_gather_stacked(out_r, group, dist)
    lses = all_gather_stacked(lse_r, group, dist)
    out, lse = ops.merge(outs, lses)
    return gidx, out, lse


def cuda_ops(dims, stream=None) -> CpOps:
    """The per-rank steps on the library's kernels.  A shard's `local` holds
    q_idx, w, k_pages, q, latent_pages (device tensors) and cache (PagedCache
    over the local keys)."""
    import torch
    import sparse_attention_scores_b200 as dsa

    def local_topk(shard, kk):
        t, cache = shard.local, shard.local["cache"]
        ld = max(4, (int(cache.max_seq_len) + 3) // 4 * 4)
        scores = torch.empty((dims.n_q, ld), dtype=torch.float32, device="cuda")
        idx = torch.empty((dims.n_q, kk), dtype=torch.int32, device="cuda")
        if "ws" not in t:
            t["ws"] = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
        ws = t["ws"]
        dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws, stream)
        dsa.dsa_topk(scores, cache.seq_lens, 0, kk, idx, ws, stream)
        return scores, idx

    def candidates(scores, idx_local, offsets):
        cs = torch.empty(idx_local.shape, dtype=torch.float32, device="cuda")
        ci = torch.empty(idx_local.shape, dtype=torch.int32, device="cuda")
        dsa.dsa_cp_candidates(scores, idx_local, offsets, cs, ci, dsa.status_workspace(), stream)
        return cs, ci

    def select(all_s, all_i, offsets, lens):
        R, n_q, kk = all_s.shape
        gidx = torch.empty((n_q, kk), dtype=torch.int32, device="cuda")
        own = torch.empty((n_q, kk), dtype=torch.int32, device="cuda")
        dsa.dsa_cp_select(all_s, all_i, offsets, lens, gidx, own, dsa.cp_workspace(R, n_q, kk),
                          stream)
        return gidx, own

    def attend(shard, own):
        t, cache = shard.local, shard.local["cache"]
        out = torch.empty((dims.n_q, dims.H, dims.R), dtype=torch.float32, device="cuda")
        lse = torch.empty((dims.n_q, dims.H), dtype=torch.float32, device="cuda")
        dsa.dsa_sparse_mla_decode(t["q"], t["latent_pages"], cache, own, dims, out, lse, t["ws"],
                                  stream)
        return out, lse

    def merge(outs, lses):
        out = torch.empty(outs.shape[1:], dtype=torch.float32, device="cuda")
        lse = torch.empty(lses.shape[1:], dtype=torch.float32, device="cuda")
        dsa.dsa_cp_merge(outs, lses, out, lse, dsa.status_workspace(), stream)
        return out, lse

    return CpOps(local_topk, candidates, select, attend, merge)
