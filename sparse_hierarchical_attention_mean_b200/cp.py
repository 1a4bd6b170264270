"""Context-parallel decode over torch.distributed ranks, one process per GPU.

Every rank holds the cache tokens [tok_lo, tok_lo + n) of every sequence and
the summaries of the blocks in that range.  One decode step (see
dash_attn_cp_scores in include/dashattn.h):

  1. this rank's routing logits into a zero-filled score buffer;
  2. a sum all-reduce of the buffer (the ranks' block ranges are disjoint);
  3. alpha-entmax, GQA mean and ascending lists from the whole scores, the
     same on every rank ("Stage 1: entmax chunk routing" needs every
     candidate of a row for its threshold, hence the exchange);
  4. stage 2 over this rank's selected blocks (and the diagonal block where
     it lies) -> partials (o, m, l) per head;
  5. an all-gather of the partials and a log-sum-exp merge.

The two collectives carry G * t_cap floats and G * (d + 2) floats per
(sequence, KV head); the K/V bytes never leave their rank.  ``ops`` supplies
the four compute steps (``CudaOps`` calls the library); the collectives come
from ``torch.distributed``.
"""

from __future__ import annotations

import torch

from . import cp_attend_ex, cp_lists, cp_merge, cp_scores


class CudaOps:
    """The compute steps on the current CUDA device, through the C ABI."""

    @staticmethod
    def zeros(shape, like):
        return torch.zeros(shape, dtype=torch.float32, device=like.device)

    @staticmethod
    def scores(q, summ, block_lo, block_hi, seqlens, lmax, alpha, block, scores):
        return cp_scores(q, summ, block_lo, block_hi, seqlens, lmax, alpha, block, scores)

    @staticmethod
    def lists(q, kv_heads, scores, seqlens, lmax, alpha, block):
        return cp_lists(q, kv_heads, scores, seqlens, lmax, alpha, block)

    @staticmethod
    def attend(q, kshard, vshard, tok_lo, seqlens, lmax, lists, block, sigma):
        # the split-KV tensor-core path (its workspace allocated per call)
        return cp_attend_ex(q, kshard, vshard, tok_lo, seqlens, lmax, lists, block, sigma)

    @staticmethod
    def merge(parts, q):
        out = torch.empty_like(q)
        return cp_merge(parts, out)


def decode_step(q, kshard, vshard, summ_shard, tok_lo: int, seqlens, lmax: int, t_cap: int, alpha: float, block: int,
                sigma: float = 1.0, ops=CudaOps, group=None):
    """One context-parallel decode step on this rank; returns out [B, 1, H, d] (the same on every rank)."""
    import torch.distributed as dist

    B, _, H, d = q.shape
    Hkv = kshard.shape[2]
    G = H // Hkv
    n = kshard.shape[1]
    assert tok_lo % block == 0 and n % block == 0
    scores = ops.zeros((B, Hkv, G, t_cap), q)
    ops.scores(q, summ_shard, tok_lo // block, (tok_lo + n) // block, seqlens, lmax, alpha, block, scores)
    dist.all_reduce(scores, op=dist.ReduceOp.SUM, group=group)
    lists = ops.lists(q, Hkv, scores, seqlens, lmax, alpha, block)
    part = ops.attend(q, kshard, vshard, tok_lo, seqlens, lmax, lists, block, sigma)
    parts = [torch.empty_like(part) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, part, group=group)
    return ops.merge(torch.stack(parts).contiguous(), q)
