// Shared pieces of the stage-2 prefill kernels: the walk over a tile's work
// list and the per-row prior bias.
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: the logits get log g added, with g = 0 (bias -inf) on blocks the
// routing gave no mass; the near-diagonal block has no summary and is always
// included, here with the uniform-baseline prior log(1/N).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace dash {

// Prior bias of one row for the tensor-core kernel (sigma * log p_bar; the
// diagonal block sigma * log(1/N)): the tile's work list carries, per block,
// the mask of tile positions that selected it, so a row only needs its own
// log p_bar values in order; they are prefetched four
// selections ahead to keep global-memory latency off the softmax path.
struct RowPrior {
  const float* lp;
  int n, cur, bit, pos, t;
  bool valid;
  float beta, sigma;
  float q0, q1, q2, q3;

  // dense prior: the work list being walked (its entry k is block ul[k])
  const int32_t* ul;

  __device__ __forceinline__ void init(const SparseParams& p, int64_t bg, int position, int pos_in_tile) {
    pos = position;
    bit = pos_in_tile;
    valid = pos < p.S;
    t = pos / p.block;
    const int n_blocks = (p.S + p.block - 1) / p.block;
    const int n_cand = p.causal ? t : n_blocks - 1;
    sigma = p.sigma;
    beta = n_cand > 0 ? sigma * logf(1.0f / (float)n_cand) : 0.0f;
    const int64_t row = bg * p.S + (valid ? pos : 0);
    n = valid ? min(max(p.cnt[row], 0), (int)p.t_cap) : 0;
    lp = p.logp + row * p.t_cap;
    ul = nullptr;
    q0 = n > 0 ? __ldg(lp) : 0.f;
    q1 = n > 1 ? __ldg(lp + 1) : 0.f;
    q2 = n > 2 ? __ldg(lp + 2) : 0.f;
    q3 = n > 3 ? __ldg(lp + 3) : 0.f;
    cur = 4;
  }
  // Dense prior (SparseParams::logp_dense): the value of block c sits at
  // column c of the row, so the queue follows the work list `list` (n_list
  // entries, ascending) instead of the row's own selections: entry k's column
  // is prefetched four entries ahead, whether or not this row selected it.
  __device__ __forceinline__ void init_dense(const SparseParams& p, int64_t bg, int position, int pos_in_tile,
                                             const int32_t* list, int n_list) {
    pos = position;
    bit = pos_in_tile;
    valid = pos < p.S;
    t = pos / p.block;
    const int n_blocks = (p.S + p.block - 1) / p.block;
    const int n_cand = p.causal ? t : n_blocks - 1;
    sigma = p.sigma;
    beta = n_cand > 0 ? sigma * logf(1.0f / (float)n_cand) : 0.0f;
    lp = p.logp_dense + (bg * p.S + (valid ? pos : 0)) * p.t_cap;
    ul = list;
    n = n_list;
    q0 = n > 0 ? __ldg(lp + __ldg(ul)) : 0.f;
    q1 = n > 1 ? __ldg(lp + __ldg(ul + 1)) : 0.f;
    q2 = n > 2 ? __ldg(lp + __ldg(ul + 2)) : 0.f;
    q3 = n > 3 ? __ldg(lp + __ldg(ul + 3)) : 0.f;
    cur = 4;
  }
  // natural-log bias of block c (-inf: masked); `mask` holds the tile
  // positions that selected c.  Called once per work-list entry, in order.
  __device__ __forceinline__ float bias(int c, const uint4& mask) {
    if (ul) {
      // dense prior: the queue advances on every entry
      const float v = q0;
      q0 = q1;
      q1 = q2;
      q2 = q3;
      q3 = cur < n ? __ldg(lp + __ldg(ul + cur)) : 0.f;
      ++cur;
      if (!valid) return kNegInf;
      if (c == t) return beta;
      const uint32_t w = bit < 32 ? mask.x : bit < 64 ? mask.y : bit < 96 ? mask.z : mask.w;
      return ((w >> (bit & 31)) & 1u) ? sigma * v : kNegInf;
    }
    if (!valid) return kNegInf;
    if (c == t) return beta;
    const uint32_t w = bit < 32 ? mask.x : bit < 64 ? mask.y : bit < 96 ? mask.z : mask.w;
    if (((w >> (bit & 31)) & 1u) == 0u) return kNegInf;
    const float v = sigma * q0;
    q0 = q1;
    q1 = q2;
    q2 = q3;
    q3 = cur < n ? __ldg(lp + cur) : 0.f;
    ++cur;
    return v;
  }
  __device__ __forceinline__ bool masked(int c, int tok, int S, int causal) const {
    return tok >= S || (causal && c == t && tok > pos);
  }
};

}  // namespace dash
