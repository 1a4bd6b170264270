// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dashattn.h"

namespace dash {

// Records the thread-local message returned by dash_attn_last_error().
dash_status_t set_last_error(dash_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

struct DeviceStatus;

// A strided [B, S, H, D] view; strides in elements, D contiguous.
struct View {
  const void* data;
  int64_t sb, ss, sh;
};

// ---------------------------------------------------------------- stage 0
struct PoolParams {
  View k;
  int dtype;  // 0 f32, 1 f16, 2 bf16
  int B, S, Hkv, D, block;
  const int32_t* seqlens;  // nullable
  const float* w_s;        // [D, D]
  const float* qbar;       // [Hkv, D] learned summary queries, or null (mean pooling)
  const int32_t* block_table;  // paged cache: block c of sequence b is page block_table[b * max_blocks + c]
  int max_blocks;              //   (k.sb = page stride, k.ss = row stride); null for a dense cache
  float* summaries;        // [B, Hkv, t_cap, D]
  int64_t t_cap;
  int64_t first_block;
};
cudaError_t launch_pool(const PoolParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- stage 1
struct RouteParams {
  View q;
  int dtype;
  int B, S, H, Hkv, G, D, block;
  int causal;
  float alpha;
  const float* summaries;  // [B, Hkv, t_cap, D]
  int64_t t_cap;
  int32_t* idx;  // [B, Hkv, S, t_cap]
  float* logp;   // [B, Hkv, S, t_cap]
  int32_t* cnt;  // [B, Hkv, S]
  float* tau;      // nullable [B, H, S]
  float* p_dense;  // nullable [B, H, S, t_cap]
  int pos_begin;   // CUDA-core kernel: first position to route (a tile boundary)
  DeviceStatus* status;  // nullable
  // tensor-core kernel: the summaries already split into tf32 head and
  // remainder in the kernel's shared-memory operand layout (route_split_bytes),
  // streamed by bulk copies; null: the kernel splits them itself
  const float* summ_split;
};
cudaError_t launch_route_prefill(const RouteParams& p, cudaStream_t stream);
// bytes of the split summaries of [B, Hkv, t_cap, D]; launch_route_split writes them
size_t route_split_bytes(int64_t B, int64_t Hkv, int64_t t_cap, int D);
cudaError_t launch_route_split(const RouteParams& p, float* split, cudaStream_t stream);

// Stage-2 work lists written by the tensor-core routing kernel (null ulist:
// not wanted).
struct TileOut {
  int32_t* ulist;
  uint4* umask;
  int32_t* ucnt;
  int32_t* usteps;
  int n_tiles;
};
// Tensor-core routing for f16/bf16 over tiles [tile0, tile0 + n_tiles) of
// 128 / G positions; every tile must have at most route_tc_max_cols() logit
// columns.
int route_tc_max_cols();
cudaError_t launch_route_prefill_tc(const RouteParams& p, const TileOut& to, int tile0, int n_tiles,
                                    cudaStream_t stream);

// Tiles with more than route_tc_max_cols() logit columns (up to
// route_tc_wide_max_cols()) run the segmented tensor-core kernel, which keeps
// each tile's logits in a scratch slot in global memory: `n_slots` slots
// (more than the SM count: one CTA of that kernel fills an SM) and one lock
// word per slot, which must be zero when the kernel starts (it leaves them
// zero).
// Needs p.summ_split.
struct WideScratch {
  float* logits;   // [n_slots][slot_floats]
  int32_t* locks;  // [n_slots]
  int n_slots;
  int64_t slot_floats;
};
int route_tc_wide_max_cols();
size_t route_wide_scratch_bytes(int64_t t_cap, int n_slots);  // locks + slots, 256-byte aligned parts
WideScratch route_wide_scratch(void* base, int64_t t_cap, int n_slots);
cudaError_t launch_route_prefill_tc_wide(const RouteParams& p, const TileOut& to, int tile0, int n_tiles,
                                         const WideScratch& w, cudaStream_t stream);

// Work list of each stage-2 tile of `tile_pos` consecutive positions: the
// union of the rows' selected blocks and the rows' own blocks, ascending.
struct UnionParams {
  int B, S, Hkv, block, tile_pos, n_tiles;
  int tile0;  // first tile to build
  int64_t t_cap;
  const int32_t* idx;
  const int32_t* cnt;
  int32_t* ulist;  // [B, Hkv, n_tiles, t_cap]
  uint4* umask;    // [B, Hkv, n_tiles, t_cap]: positions of the tile that selected the block
  int32_t* ucnt;   // [B, Hkv, n_tiles]
  int32_t* usteps; // [B, Hkv, n_tiles]: 64-token steps of the tile
  int causal;
  DeviceStatus* status;  // invalid list entries are skipped and reported here
  // bit-packed form instead of idx / cnt (non-null: used): [B, Hkv, S, n_words],
  // bit c of a row set iff block c is selected
  const uint32_t* mask;
  int n_words;
};
cudaError_t launch_union(const UnionParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- stage 2
struct SparseParams {
  View q, k, v, out;
  int dtype;
  int B, S, H, Hkv, G, D, block;
  int causal;
  int64_t t_cap;
  const int32_t* idx;
  const float* logp;
  const int32_t* cnt;
  const int32_t* plist;  // work lists of tile pairs (tensor-core kernel)
  const uint4* pmask;    // [.., t_cap, 2]: per block, the selecting positions of each tile
  const int32_t* pcnt;
  const int32_t* psteps;
  int tile_pos, n_tiles, n_pairs;
  float sigma;  // prior strength: bias sigma * log p_bar (diagonal: sigma * log(1/N))
  DeviceStatus* status;
  // dense prior instead of the lists (tensor-core kernel; non-null: used):
  // [B, Hkv, S, t_cap], log p_bar of block c at column c, read only where the
  // tile work list marks the row as selecting c
  const float* logp_dense;
  // test of the timeout path (tensor-core kernel): cycles a consumer waits for
  // a hand-off before it gives up (0: the default, about a second), and a
  // switch that makes the producer issue no copies, so every consumer wait
  // runs out.  Waits that drain issued copies or MMAs always use the default.
  long long wait_cycles;
  int stall_producer;
  // tensor-core kernel: per-row log-sum-exp of the biased logits in log2
  // units, [B, H, S] (null: not written); skip_out: do not write `out`
  float* lse;
  int skip_out;
};
// positions per stage-2 tile (tiles are 128 rows)
int sparse_tile_positions(int G, int block);
// tiles per CTA of the tensor-core stage-2 kernel
int sparse_tile_pair();

// Work list of each pair of adjacent tiles: the union of the two tiles'
// lists, each block with both tiles' position masks, and the pair's number
// of 64-token steps.
struct PairParams {
  int B, S, Hkv, block, tile_pos, n_tiles, n_pairs, causal;
  int64_t t_cap;
  const int32_t* ulist;
  const uint4* umask;
  const int32_t* ucnt;
  int32_t* plist;
  uint4* pmask;
  int32_t* pcnt;
  int32_t* psteps;
};
cudaError_t launch_pairs(const PairParams& p, cudaStream_t stream);
// 4-D TMA map over a [B, S, H, D] f16/bf16 view (innermost first: D, H, S,
// B), 128-byte swizzle, box {64, box_h, box_s, 1}; no multicast.
bool make_map(CUtensorMap* map, const View& v, int dtype, int64_t B, int64_t S, int64_t H, int D, int box_h,
              int box_s);
cudaError_t launch_sparse_prefill(const SparseParams& p, cudaStream_t stream);
cudaError_t launch_sparse_prefill_tc(const SparseParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- decode
struct DecodeParams {
  View q, k, v, out;
  int dtype;
  int B, Lmax, H, Hkv, G, D, block;
  float alpha;
  const int32_t* seqlens;
  const float* summaries;
  int64_t t_cap;
  // workspace
  float* scores;     // [B, Hkv, G, t_cap]
  int32_t* idx;      // [B, Hkv, t_cap]
  float* logp;       // [B, Hkv, t_cap]
  int32_t* cnt;      // [B, Hkv]
  int32_t* items;    // [max_items] packed work items
  int32_t* n_items;  // device counter
  int32_t* pair_base;  // [B, Hkv]
  float* part_o;     // [max_items, G, D]
  float* part_ml;    // [max_items, G, 2]
  int64_t max_items;
  int chunk_blocks;  // selected blocks per split-KV work item
  float sigma;       // prior strength (as in SparseParams)
  // context parallelism: this shard scores blocks [c_lo, c_hi) whose summaries
  // sit at index c - c_lo of `summaries` (capacity summ_cap blocks); the
  // whole-context decode uses c_lo = 0, c_hi = t_cap, summ_cap = t_cap
  int c_lo, c_hi;
  int64_t summ_cap;
  // shard attention: cache tokens [tok_lo, tok_lo + k.s) of every sequence,
  // partials [B, H, D + 2] (o relative to m, m in log2 units, l)
  int tok_lo, tok_n;
  float* part;
  // paged cache (split-KV decode): block c of sequence b is page
  // block_table[b * max_blocks + c] of k / v (sb = page stride); null: dense
  const int32_t* block_table;
  int max_blocks;
  // split-KV attention over one shard of the cache (context parallelism):
  // per (b, g) four ints {first list entry, end entry, diagonal held, items};
  // the shard's k / v rows start at token tok_lo.  Null: the whole list and
  // the diagonal block (the regular decode step).
  int32_t* shard;
  // optional route outputs (dash_attn_route in decode mode)
  float* tau;      // [B, H]
  float* p_dense;  // [B, H, t_cap]
  DeviceStatus* status;
};
int64_t decode_max_items(int64_t B, int64_t Hkv, int64_t t_cap, int chunk_blocks);
cudaError_t launch_decode_route(const DecodeParams& p, cudaStream_t stream);
// bit-packed active-block masks from ascending lists: rows x n_words uint32
cudaError_t launch_lists_to_mask(const int32_t* idx, const int32_t* cnt, int64_t rows, int64_t t_cap,
                                 uint32_t* mask, int n_words, cudaStream_t stream);
cudaError_t launch_decode_attend(const DecodeParams& p, int num_sms, cudaStream_t stream);
// context parallelism: shard scores (score kernel only), lists from a score
// buffer (entmax kernel without work items), shard attention, partial merge
cudaError_t launch_cp_scores(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_cp_lists(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_cp_attend(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_cp_merge(const float* parts, int n_parts, int B, int H, int D, const View& out, int dtype,
                            cudaStream_t stream);
// context parallelism on the split-KV tensor-core path: the shard's work
// items (p.shard, p.items, p.n_items zeroed, p.pair_base), the split-KV
// kernel over them and a combine into per-head partials p.part [B, H, D + 2]
cudaError_t launch_cp_attend_mma(const DecodeParams& p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- backward
// Gradients of sum(dout * out) for the prefill forward (f16/bf16 inputs,
// fp32 gradients).  The summaries, lists and thresholds are the forward's,
// recomputed by the caller before the four kernels run in order:
//   row    (query block, head): LSE, dq of stage 2, d log p_bar per head
//   route  (row, KV head): entmax vector-Jacobian product, dq of stage 1
//   key    (key block, KV head): dk, dv of stage 2, the summary gradient and
//          its stage-0 projection into dk
//   ws     dW_s = sum over blocks of kbar^T ds
struct BwdParams {
  View q, k, v, o, dout;  // [B, S, H or Hkv, D], dtype
  View dq, dk, dv;        // fp32, same shapes
  int dtype;
  int B, S, H, Hkv, G, D, block, causal;
  float alpha, sigma;
  const float* w_s;        // [D, D]
  const float* summaries;  // [B, Hkv, t_cap, D]
  int64_t t_cap;           // ceil(S / block)
  int n_qblocks;           // ceil(S / block)
  int n_words;             // ceil(t_cap / 32)
  const int32_t* idx;      // [B, Hkv, S, t_cap]
  const float* logp;       // [B, Hkv, S, t_cap]
  const int32_t* cnt;      // [B, Hkv, S]
  const float* tau;        // [B, H, S]
  const float* lse;        // [B, H, S] log-sum-exp of the logits, log2 units (from the forward kernel)
  float* dd;               // [B, H, S] dout . out
  float* dz;               // [B, Hkv, S, t_cap, G]: d log p_bar per head, then dL/dz
  uint32_t* umask;         // [B, Hkv, n_qblocks, n_words]: blocks some row of the query block selected
  float* kbar;             // [B, Hkv, t_cap, D] block means
  float* ds;               // [B, Hkv, t_cap, D] dL/d(summary)
  float* dw_s;             // [D, D]
  DeviceStatus* status;
  // key-centric tensor-core kernel: the stage-2 tiles (128 / G positions x G
  // heads) whose work lists hold each block, and each row's selection
  const uint32_t* tbits;   // [B, Hkv, n_tiles, n_words]: bit c set iff block c is in the tile's work list
  const uint32_t* rmask;   // [B, Hkv, S, n_words]: bit c set iff the row selected block c
  const int32_t* rrank;    // [B, Hkv, S, n_words]: the row's selections below block 32 w
  int n_tiles;
  // row-centric tensor-core kernel: the stage-2 tiles' work lists ([B, Hkv, n_tiles] lists of
  // t_cap entries: blocks ascending, the mask of tile positions that selected each, counts, steps)
  const int32_t* ulist;
  const uint4* tmask;
  const int32_t* ucnt;
  const int32_t* usteps;
};
cudaError_t launch_bwd(const BwdParams& p, cudaStream_t stream);
// the key-centric backward kernel alone (dk, dv, ds, kbar), and the tile bit
// masks it reads, from the tiles' work lists ulist / ucnt ([n_lists][t_cap])
cudaError_t launch_bwd_key_tc(const BwdParams& p, cudaStream_t stream);
// the row-centric backward kernel alone (dq of stage 2, d log p_bar per head into dz, D into dd)
cudaError_t launch_bwd_row_tc(const BwdParams& p, cudaStream_t stream);
cudaError_t launch_row_ranks(const uint32_t* mask, int64_t rows, int n_words, int32_t* rank, cudaStream_t stream);
cudaError_t launch_tile_bits(const int32_t* ulist, const int32_t* ucnt, int64_t n_lists, int64_t t_cap, uint32_t* bits,
                             int n_words, cudaStream_t stream);

}  // namespace dash
