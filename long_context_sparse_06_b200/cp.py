"""Context-parallel decode of long requests: one process per GPU, torch.distributed for the
exchange ("DeepSeek V4 深度解析" §2, CSA steps 2-3, split over shards of the compressed entries).

Every rank holds a contiguous shard [offset, offset + S) of each request's compressed KV rows
and index keys; the rank that holds the newest raw tokens also holds the window rows.  One
decode step on every rank:

1. index scores and the top-k of its own shard (local indices), turned into
   (score, global index) candidates;
2. one all-gather of the candidates, in rank order -- that is global-index order, so the
   global top-k of the candidates is the unsplit top-k with the same tie rule;
3. the global selection and this rank's share of it (local indices);
4. attention over that share (and the window, on its rank), normalised output and
   log-sum-exp per head;
5. one all-gather of those partials and their log-sum-exp merge.

The arithmetic runs in liblcs's kernels (``LibOps``); this module only moves tensors between
ranks and calls them.  The phases are separate functions so that a caller (or a test) can run
them for several ranks in one process.
"""
from __future__ import annotations

import long_context_sparse_06_b200 as L


class LibOps:
    """The library calls of one rank (CUDA tensors)."""

    def __init__(self, kv_dtype=None, kI_dtype=None, score_dtype=None):
        self.kv_dtype, self.kI_dtype, self.score_dtype = kv_dtype, kI_dtype, score_dtype

    def index_topk(self, qI, w, kI, k, N_c):
        B, HI, DI = qI.shape
        idx, scores = L.csa_index_topk(qI.view(B, 1, HI, DI), w.view(B, 1, HI), kI, k, N_c=N_c,
                                       kI_dtype=self.kI_dtype, score_dtype=self.score_dtype, want_scores=True)
        return idx.view(B, k), scores.view(B, N_c)

    def candidates(self, scores, idx, offset):
        return L.lcs_cp_candidates(scores, idx, offset)

    def select(self, cand_score, cand_idx, offset, S):
        return L.lcs_cp_select(cand_score, cand_idx, offset, S)

    def attend(self, q, comp, win, idx_local, d_v, scale):
        import torch
        B, H, D = q.shape
        k = idx_local.shape[-1]
        o, lse = L.csa_attend(q.view(B, 1, H, D), comp, win, idx_local.view(B, 1, k), d_v, scale,
                              kv_dtype=self.kv_dtype, want_lse=True, out_dtype=torch.float32)
        return o.view(B, H, d_v), lse.view(B, H)

    def merge(self, o, lse, out_dtype):
        return L.lcs_attn_merge(o, lse, out_dtype=out_dtype)


def local_candidates(ops, qI, w, kI, k, offset, S):
    """Phase 1: this rank's top-k as (score, global index) candidates [B, k]."""
    idx, scores = ops.index_topk(qI, w, kI, k, S)
    return ops.candidates(scores, idx, offset)


def local_attention(ops, q, comp, win, cand_score, cand_idx, offset, S, d_v, scale):
    """Phases 3-4: from all ranks' candidates [G, B, k], the global selection [B, k] and this
    rank's attention partial (o [B, H, d_v] fp32, lse [B, H])."""
    idx_global, idx_local = ops.select(cand_score, cand_idx, offset, S)
    o, lse = ops.attend(q, comp, win, idx_local, d_v, scale)
    return idx_global, o, lse


def _all_gather(t, world, group):
    """[world, *t.shape]: every rank's t, in rank order."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def cp_decode_step(q, comp, win, qI, w, kI, k, offset, d_v, scale, group=None, ops=None, out_dtype=None):
    """One decode step of B requests whose entries are split over the ranks of `group`.

    q [B, H, D], qI [B, H_I, d_I], w [B, H_I]: this step's queries (the same on every rank);
    comp [B, S, row], kI [B, S, d_I] (or FP4 planes): this rank's shard, global entries
    [offset, offset + S); win [B, Tw, row] on the rank holding the window, else None.
    Returns (out [B, H, d_v], the global selection [B, k]) on every rank."""
    import torch.distributed as dist
    ops = ops or LibOps()
    world = dist.get_world_size(group)
    S = comp.shape[1]
    cs, ci = local_candidates(ops, qI, w, kI, k, offset, S)
    cs_all, ci_all = _all_gather(cs, world, group), _all_gather(ci, world, group)
    idx_global, o, lse = local_attention(ops, q, comp, win, cs_all, ci_all, offset, S, d_v, scale)
    o_all, lse_all = _all_gather(o, world, group), _all_gather(lse, world, group)
    out = ops.merge(o_all, lse_all, out_dtype or q.dtype)
    return out, idx_global
