/*
 * dashattn.h -- C ABI of libdashattn, the B200 (sm_100a) forward and
 * backward of DashAttention sparse hierarchical attention.
 *
 * Source of the method: "DashAttention: Differentiable and Adaptive Sparse
 * Hierarchical Attention" (gist.science explainer of arXiv 2605.18753),
 * technical summary, sections "Stage 0: local chunk summary",
 * "Stage 1: entmax chunk routing" and "Stage 2: prior-induced sparse
 * softmax".  alpha-entmax as in Peters, Niculae & Martins (2019).
 *
 * What the library computes, per batch element b and KV head g (G = H/Hkv
 * query heads share g), for a query at position pos in block t = pos / B:
 *   stage 0  s_c = mean_{j in block c} k_j @ W_s                 (fp32)
 *   stage 1  z_{h,c} = q_h . s_c / sqrt(d);  p_h = alpha-entmax(z_h) over the
 *            N candidate blocks (causal: the complete blocks c < t);
 *            p_bar = mean over the G heads; selected = {c : p_bar_c > 0}
 *   stage 2  o_h = sum_j softmax_j(q_h . k_j / sqrt(d) + bias_j) v_j over the
 *            tokens of the selected blocks (bias log p_bar_c) and of the
 *            diagonal block t (tokens <= pos when causal; bias log(1/N),
 *            0 when N = 0).
 *
 * Conventions shared by every entry point
 *  - Tensors are described by dash_tensor_t: a DEVICE pointer with extents
 *    (b, s, h, d) and element strides for b, s and h; the d dimension is
 *    contiguous.  Base pointers and the b/s/h strides (in bytes) must be
 *    multiples of 16 bytes.  q and out are [B, S, H, d]; k and v are
 *    [B, S, Hkv, d] (FlashAttention layout).
 *  - q, k and v share one dtype: DASH_F32, DASH_F16 or DASH_BF16.  f16/bf16
 *    use tensor cores with fp32 accumulation; f32 runs an fp32 CUDA-core
 *    path.  Summaries, routing weights and thresholds are always fp32.
 *  - Supported: d in {64, 128}; block in {64, 128}; G = H / Hkv in
 *    {1, 2, 4, 8}; 1 < alpha <= 2.
 *  - Ownership: the caller allocates every buffer (inputs, outputs,
 *    workspace) and keeps it alive until the stream work completes.  The
 *    library allocates no memory.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) of the current device; nothing synchronises.
 *  - Errors: invalid arguments are detected on the host before anything is
 *    launched and return a non-zero dash_status_t; dash_attn_last_error()
 *    then gives a message (thread-local).  A failed launch returns
 *    DASH_ERR_CUDA.  Device-side waits are bounded: if one gives up, the
 *    kernel records DASH_ERR_DEVICE_TIMEOUT in the workspace status word,
 *    which dash_attn_get_device_status() reads.
 */
#ifndef DASHATTN_H_
#define DASHATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dash_stream_t; /* same handle as cudaStream_t */

typedef enum {
  DASH_OK = 0,
  DASH_ERR_INVALID_ARGUMENT = 1,
  DASH_ERR_UNSUPPORTED = 2,
  DASH_ERR_WORKSPACE_TOO_SMALL = 3,
  DASH_ERR_CUDA = 4,
  DASH_ERR_DEVICE_TIMEOUT = 5
} dash_status_t;

typedef enum { DASH_F32 = 0, DASH_F16 = 1, DASH_BF16 = 2 } dash_dtype_t;

typedef struct {
  void* data;     /* device pointer to element (0, 0, 0, 0) */
  int32_t dtype;  /* dash_dtype_t */
  int32_t reserved;
  int64_t b, s, h, d;                   /* extents */
  int64_t stride_b, stride_s, stride_h; /* element strides; d is contiguous */
} dash_tensor_t;

/* Library version, major * 10000 + minor * 100 + patch. */
int dash_attn_version(void);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* dash_attn_last_error(void);

/*
 * Bytes of workspace dash_attn_fwd needs for q [B, S, H, d], k [B, S, Hkv, d]
 * and `block`.  Holds the stage-0 summaries [B, Hkv, T, d] fp32 (T =
 * ceil(S / block)), the per-row routing lists [B, Hkv, S, T] (int32 block
 * ids and fp32 log p_bar), the counts [B, Hkv, S], the per-tile union lists
 * and a status word.  Returns 0 for arguments dash_attn_fwd would reject.
 */
size_t dash_attn_fwd_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block);

/*
 * Where a dash_attn_fwd / dash_attn_fwd_ex call leaves its stage-0 summaries
 * and routing lists in its workspace (same q, k and block as the call): byte
 * offsets from the workspace base of
 *   summaries [B, Hkv, T, d] fp32,
 *   idx       [B, Hkv, S, T] int32, each row's selected block ids ascending,
 *   logp      [B, Hkv, S, T] fp32, log p_bar of those blocks,
 *   cnt       [B, Hkv, S] int32, the number of valid entries of each row,
 * with T = ceil(S / block).  Entries of idx / logp past cnt are undefined.
 * Any offset pointer may be NULL.  Host-only; launches nothing.
 */
dash_status_t dash_attn_fwd_workspace_lists(const dash_tensor_t* q, const dash_tensor_t* k, int block,
                                            size_t* summ_offset, size_t* idx_offset, size_t* logp_offset,
                                            size_t* cnt_offset);

/*
 * Full prefill forward: stages 0, 1 and 2 ("Stage 0" to "Stage 2" of the
 * cited technical summary) over q [B, S, H, d], k, v [B, S, Hkv, d].
 *   w_s       device fp32 [d, d] row-major; summaries are mean(k) @ w_s.
 *   alpha     entmax alpha, 1 < alpha <= 2.
 *   block     block (chunk) size B, 64 or 128.
 *   causal    1: candidates are the complete blocks before the query's own
 *             block, which is included with a causal mask.  0: every other
 *             block is a candidate (a trailing partial block is pooled over
 *             its valid tokens) and the own block is included whole.
 *   out       [B, S, H, d], same dtype as q; written once per element.
 *   workspace device buffer of at least dash_attn_fwd_workspace_size()
 *             bytes, 256-byte aligned; on return it holds the call's
 *             summaries and routing lists, at the offsets that
 *             dash_attn_fwd_workspace_lists gives.
 */
dash_status_t dash_attn_fwd(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                            const float* w_s, float alpha, int block, int causal, dash_tensor_t* out,
                            void* workspace, size_t workspace_bytes, dash_stream_t stream);

/*
 * Stage 0 alone ("Stage 0: local chunk summary"; a summary is fixed and
 * cached once its chunk is complete): summaries[b, g, c, :] =
 * mean_{j in block c, j < n_b} k[b, j, g, :] @ w_s for blocks
 * first_block <= c < ceil(n_b / block), where n_b = seqlens[b] (or k->s when
 * seqlens is NULL).  A trailing partial block is averaged over its valid
 * tokens; a decode step never reads it (it is the query's diagonal block).
 *   seqlens         device int32 [B] or NULL.
 *   summaries       device fp32 [B, Hkv, t_cap, d], contiguous.
 *   t_cap           block capacity of `summaries`; must be >= ceil(k->s / block).
 *   first_block     first block to (re)compute; 0 for all.  Decoding calls
 *                   this again with the first block that has just completed.
 */
dash_status_t dash_attn_summarize(const dash_tensor_t* k, const int32_t* seqlens, const float* w_s,
                                  int block, float* summaries, int64_t t_cap, int64_t first_block,
                                  dash_stream_t stream);

/*
 * Stage 0 with the learned summary query ("Stage 0: local chunk summary":
 * a learned query vector attends to the keys of each chunk through local
 * scaled dot-product attention; initialised at zero it is uniform mean
 * pooling).  Same as dash_attn_summarize, with the mean replaced by
 *   sum_j softmax_j(qbar[g] . k[b, j, g, :] / sqrt(d)) k[b, j, g, :]
 * over the block's valid tokens, then @ w_s.
 *   qbar  device fp32 [Hkv, d], one query per KV head, 16-byte aligned, or
 *         NULL (then identical to dash_attn_summarize).
 * Errors and the other arguments as for dash_attn_summarize.
 */
dash_status_t dash_attn_summarize_sdpa(const dash_tensor_t* k, const int32_t* seqlens, const float* w_s,
                                       const float* qbar, int block, float* summaries, int64_t t_cap,
                                       int64_t first_block, dash_stream_t stream);

/*
 * Options of the variants the pages name beside the path the spec fixes.
 * Pass NULL for the defaults (sigma = 1, mean pooling).
 *   sigma  strength of the prior ("Stage 2: prior-induced sparse softmax"
 *          names a strength that balances the prior against the uniform
 *          baseline): the stage-2 bias is sigma * log p_bar on a selected
 *          block and sigma * log(1/N) on the diagonal block, so a uniform
 *          prior is full attention for every sigma and sigma = 0 is plain
 *          softmax over the selected tokens.  Finite, >= 0.
 *   qbar   learned summary queries, device fp32 [Hkv, d], 16-byte aligned,
 *          or NULL: stage 0 as dash_attn_summarize_sdpa.  Only the prefill
 *          forward computes summaries; the other calls reject a non-NULL qbar.
 */
typedef struct {
  float sigma;
  const float* qbar;
} dash_options_t;

/* dash_attn_fwd with options (opts may be NULL). */
dash_status_t dash_attn_fwd_ex(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                               const float* w_s, float alpha, int block, int causal, dash_tensor_t* out,
                               void* workspace, size_t workspace_bytes, const dash_options_t* opts,
                               dash_stream_t stream);

/*
 * Backward pass of the prefill forward (dash_attn_fwd_ex with the same
 * arguments): the gradients of sum(dout * out) with respect to q, k, v and
 * W_s.  "Stage 1: entmax chunk routing" of the cited technical summary makes
 * the router differentiable, so the loss reaches W_s and q through the
 * prior log p_bar: per query row and KV group,
 *   stage 2   dS_j = P_j (dout . v_j - dout . out); dq, dk, dv as in softmax
 *             attention; d log p_bar_c = sigma * sum_{j in c, heads} dS_j
 *   routing   dp_h = d log p_bar / (G p_bar);  dz_h = u (dp_h - <u, dp_h> / sum u)
 *             with u = p_h^(2 - alpha) on the support (the alpha-entmax
 *             Jacobian, Peters, Niculae & Martins 2019, section 3)
 *   scores    dq_h += dz_h S / sqrt(d);  ds_c += dz_{h,c} q_h / sqrt(d)
 *   stage 0   dW_s = sum_c kbar_c^T ds_c;  dk_j += ds_c W_s^T / |c| for j in c.
 * The diagonal block's prior is a constant.  Stage 0 is mean pooling
 * (opts->qbar must be NULL); opts->sigma is the forward's prior strength.
 *   q, k, v, w_s, alpha, block, causal  as for dash_attn_fwd; dtype f16 or bf16
 *             (DASH_F32 inputs return DASH_ERR_UNSUPPORTED).
 *   out       the forward's output [B, S, H, d], dtype of q.
 *   dout      dL/dout [B, S, H, d], dtype of q.
 *   dq        fp32 [B, S, H, d]; dk, dv fp32 [B, S, Hkv, d]; every element
 *             is overwritten.
 *   dw_s      device fp32 [d, d], overwritten.
 *   workspace at least dash_attn_bwd_workspace_size() bytes, 256-byte
 *             aligned: summaries, routing lists and thresholds (recomputed
 *             here), row statistics, per-head routing gradients
 *             [B, Hkv, S, T, G] fp32, block means and summary gradients.
 * Arithmetic: the three attention products of each tile run as bf16/f16
 * tensor-core MMAs with fp32 accumulation (P and dS are rounded to the input
 * type as MMA operands); the routing gradient is fp32.
 */
size_t dash_attn_bwd_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block);
dash_status_t dash_attn_bwd(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                            const float* w_s, const dash_tensor_t* out, const dash_tensor_t* dout, float alpha,
                            int block, int causal, const dash_options_t* opts, dash_tensor_t* dq, dash_tensor_t* dk,
                            dash_tensor_t* dv, float* dw_s, void* workspace, size_t workspace_bytes,
                            dash_stream_t stream);

/*
 * Paged KV cache (the layout of serving engines): the cache is a pool of
 * pages of `block` tokens, k_pages / v_pages [n_pages, block, Hkv, d]
 * (dash_tensor_t with b = n_pages, s = block), and block c of sequence b
 * lives in page block_table[b * max_blocks + c] (device int32
 * [batch, max_blocks]; entries past a sequence's blocks are not read).  The
 * context bound is lmax = max_blocks * block.  Results are those of
 * dash_attn_summarize_sdpa / dash_attn_decode_ex on the same cache laid out
 * densely.  The decode workspace is dash_attn_decode_workspace_size of a
 * dense cache with the same B, Hkv and d.
 */
dash_status_t dash_attn_summarize_paged(const dash_tensor_t* k_pages, const int32_t* block_table, int64_t max_blocks,
                                        int64_t batch, const int32_t* seqlens, const float* w_s, const float* qbar,
                                        int block, float* summaries, int64_t t_cap, int64_t first_block,
                                        dash_stream_t stream);
dash_status_t dash_attn_decode_paged(const dash_tensor_t* q, const dash_tensor_t* k_pages, const dash_tensor_t* v_pages,
                                     const int32_t* block_table, int64_t max_blocks, const int32_t* seqlens,
                                     const float* summaries, int64_t t_cap, float alpha, int block, dash_tensor_t* out,
                                     void* workspace, size_t workspace_bytes, const dash_options_t* opts,
                                     dash_stream_t stream);

/*
 * Context-parallel decode: one sequence's context split over R ranks (one
 * process per GPU), each holding the cache tokens [tok_lo, tok_lo + n) of
 * every sequence (tok_lo and n multiples of the block) and the summaries of
 * the blocks in that range.  The result equals dash_attn_decode on the whole
 * cache.  One step, on every rank:
 *   1. dash_attn_cp_scores: the routing logits of this rank's candidate
 *      blocks into a zero-filled score buffer [B, Hkv, G, t_cap] fp32;
 *   2. a sum all-reduce of that buffer over the ranks (the ranges are
 *      disjoint, so the sum is the whole score vector);
 *   3. dash_attn_cp_lists: alpha-entmax, GQA mean and ascending lists, the
 *      same on every rank;
 *   4. dash_attn_cp_attend: stage 2 over this rank's selected blocks and, if
 *      it holds it, the diagonal block -> partials [B, H, d + 2] fp32 (o
 *      relative to its reference max m, m in log2 units, l);
 *   5. an all-gather of the partials ([R, B, H, d + 2]) and dash_attn_cp_merge.
 * q is [B, 1, H, d] (f16/bf16), seqlens device int32 [B] with
 * 1 <= seqlens[b] <= lmax, t_cap >= ceil(lmax / block), at most 4096.
 *   summaries  this rank's summaries, block c at index c - block_lo of a
 *              [B, Hkv, summ_cap, d] fp32 buffer (dash_attn_summarize on the
 *              shard); block_lo <= c < block_hi are scored.
 */
dash_status_t dash_attn_cp_scores(const dash_tensor_t* q, int64_t kv_heads, const float* summaries, int64_t summ_cap,
                                  int64_t block_lo, int64_t block_hi, const int32_t* seqlens, int64_t lmax, float alpha,
                                  int block, float* scores, int64_t t_cap, dash_stream_t stream);
dash_status_t dash_attn_cp_lists(const dash_tensor_t* q, int64_t kv_heads, const float* scores, const int32_t* seqlens,
                                 int64_t lmax, float alpha, int block, int32_t* idx, float* logp, int32_t* cnt,
                                 int64_t t_cap, dash_stream_t stream);
/*   kshard, vshard  [B, n, Hkv, d]: cache tokens tok_lo .. tok_lo + n - 1.
 *   opts            NULL or sigma only (opts->qbar must be NULL). */
dash_status_t dash_attn_cp_attend(const dash_tensor_t* q, const dash_tensor_t* kshard, const dash_tensor_t* vshard,
                                  int64_t tok_lo, const int32_t* seqlens, int64_t lmax, const int32_t* idx,
                                  const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                  const dash_options_t* opts, float* part, dash_stream_t stream);
/*
 * dash_attn_cp_attend_ex: step 4 on the tensor-core split-KV path of
 * dash_attn_decode_ex.  Same arguments and partials as dash_attn_cp_attend;
 * the range of each (b, KV head)'s ascending list that falls in the shard's
 * blocks, plus the diagonal block when the shard holds it, is cut into work
 * items that the whole GPU shares.  Partials are the same up to rounding
 * order.
 *   workspace  256-byte aligned device pointer of at least
 *              dash_attn_cp_attend_workspace_size(B, H, Hkv, d, block, t_cap)
 *              bytes, owned by the caller; the call may use it until the
 *              stream reaches its end.  Too small: DASH_ERR_WORKSPACE_TOO_SMALL.
 * dash_attn_cp_attend_workspace_size returns 0 for invalid sizes.
 */
size_t dash_attn_cp_attend_workspace_size(int64_t batch, int64_t heads, int64_t kv_heads, int64_t head_dim, int block,
                                          int64_t t_cap);
dash_status_t dash_attn_cp_attend_ex(const dash_tensor_t* q, const dash_tensor_t* kshard, const dash_tensor_t* vshard,
                                     int64_t tok_lo, const int32_t* seqlens, int64_t lmax, const int32_t* idx,
                                     const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                     const dash_options_t* opts, float* part, void* workspace, size_t workspace_bytes,
                                     dash_stream_t stream);
/*   parts  device fp32 [n_parts, B, H, d + 2]; out [B, 1, H, d] (f16/bf16). */
dash_status_t dash_attn_cp_merge(const float* parts, int64_t n_parts, dash_tensor_t* out, dash_stream_t stream);

/*
 * Bit-packed active-block masks from routing lists (the pages' kernel walks
 * a mask of the active chunks; the lists of dash_attn_route carry the same
 * sets plus log p_bar): for each of `rows` rows (e.g. B * Hkv * S of the
 * route layout), word w of mask[row] has bit b set iff block 32 w + b is
 * among idx[row, 0 .. cnt[row]).
 *   idx      device int32 [rows, t_cap]; cnt device int32 [rows].
 *   mask     device uint32 [rows, n_words], fully written.
 *   n_words  words per row, n_words * 32 >= t_cap, at most 128.
 */
dash_status_t dash_attn_lists_to_mask(const int32_t* idx, const int32_t* cnt, int64_t rows, int64_t t_cap,
                                      uint32_t* mask, int64_t n_words, dash_stream_t stream);

/*
 * Bytes of workspace dash_attn_decode needs for q [B, 1, H, d] against a KV
 * cache [B, Lmax, Hkv, d] with summaries of capacity t_cap blocks.
 */
size_t dash_attn_decode_workspace_size(const dash_tensor_t* q, const dash_tensor_t* kcache, int block,
                                       int64_t t_cap);

/*
 * Where a dash_attn_decode / dash_attn_decode_ex call leaves the routing of
 * its step in its workspace (same q, kcache, block and t_cap as the call):
 * byte offsets of idx [B, Hkv, t_cap] int32 (ascending), logp
 * [B, Hkv, t_cap] fp32 and cnt [B, Hkv] int32.  Any pointer may be NULL.
 * Host-only; launches nothing.
 */
dash_status_t dash_attn_decode_workspace_lists(const dash_tensor_t* q, const dash_tensor_t* kcache, int block,
                                               int64_t t_cap, size_t* idx_offset, size_t* logp_offset,
                                               size_t* cnt_offset);

/*
 * One decode step (stages 1 and 2 for a single new query token per
 * sequence; "supports prefill and incremental decoding" in the cited
 * technical summary).  The query of sequence b sits at position
 * pos = seqlens[b] - 1; its candidates are the complete blocks
 * c < pos / block, read from the cached summaries; the diagonal block holds
 * tokens [ (pos / block) * block, pos ].
 *   q          [B, 1, H, d]; kcache, vcache [B, Lmax, Hkv, d] (same dtype).
 *   seqlens    device int32 [B], 1 <= seqlens[b] <= Lmax.
 *   summaries  device fp32 [B, Hkv, t_cap, d] from dash_attn_summarize.
 *   out        [B, 1, H, d].
 */
dash_status_t dash_attn_decode(const dash_tensor_t* q, const dash_tensor_t* kcache, const dash_tensor_t* vcache,
                               const int32_t* seqlens, const float* summaries, int64_t t_cap, float alpha,
                               int block, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                               dash_stream_t stream);

/* dash_attn_decode with options (opts may be NULL; opts->qbar must be NULL). */
dash_status_t dash_attn_decode_ex(const dash_tensor_t* q, const dash_tensor_t* kcache, const dash_tensor_t* vcache,
                                  const int32_t* seqlens, const float* summaries, int64_t t_cap, float alpha,
                                  int block, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                  const dash_options_t* opts, dash_stream_t stream);

/*
 * Stage 1 alone ("Stage 1: entmax chunk routing", including GQA handling),
 * for parity checks and for callers that bring their own stage 2.
 * Prefill mode (seqlens == NULL): q is [B, S, H, d], the query at row i sits
 * at position i and the context holds S tokens.  Decode mode: q is
 * [B, 1, H, d] and the query of sequence b sits at seqlens[b] - 1 (always
 * causal; seqlens[b] <= t_cap * block).
 *   summaries  device fp32 [B, kv_heads, t_cap, d].
 *   idx, logp  device [B, kv_heads, Sq, t_cap]: for each query row the
 *              selected block ids in ascending order and log p_bar of each;
 *              entries past cnt are left untouched.
 *   cnt        device int32 [B, kv_heads, Sq]: number of selected blocks.
 *   tau        optional device fp32 [B, H, Sq]: entmax threshold of each
 *              head on the (alpha - 1) * z scale (0 when N = 0).
 *   p_dense    optional device fp32 [B, H, Sq, t_cap]: per-head entmax
 *              weight of every block (0 for non-candidates).
 *   workspace  decode mode: dash_attn_route_workspace_size(..., 1) bytes,
 *              256-byte aligned (the per-head logits).  Prefill mode: NULL,
 *              or dash_attn_route_workspace_size(..., 0) bytes, 256-byte
 *              aligned, where the f16/bf16 path keeps the summaries split
 *              for the tensor cores (same results, faster).
 */
size_t dash_attn_route_workspace_size(const dash_tensor_t* q, int64_t kv_heads, int64_t t_cap, int decode);

dash_status_t dash_attn_route(const dash_tensor_t* q, const float* summaries, int64_t kv_heads, int64_t t_cap,
                              const int32_t* seqlens, float alpha, int block, int causal, int32_t* idx,
                              float* logp, int32_t* cnt, float* tau, float* p_dense, void* workspace,
                              size_t workspace_bytes, dash_stream_t stream);

/*
 * Bytes of workspace dash_attn_sparse needs (per-tile union lists and a
 * status word).
 */
size_t dash_attn_sparse_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block, int64_t t_cap);

/*
 * Stage 2 alone ("Stage 2: prior-induced sparse softmax") on caller-given
 * routing in the layout dash_attn_route writes (idx/logp/cnt with block
 * capacity t_cap).  The diagonal block is always added with bias log(1/N).
 * Selecting every candidate with logp = log(1/N) reproduces full attention.
 */
dash_status_t dash_attn_sparse(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                               const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap,
                               int block, int causal, dash_tensor_t* out, void* workspace,
                               size_t workspace_bytes, dash_stream_t stream);

/* dash_attn_sparse with options (opts may be NULL; opts->qbar must be NULL). */
dash_status_t dash_attn_sparse_ex(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                  const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                  int causal, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                  const dash_options_t* opts, dash_stream_t stream);

/*
 * Stage 2 on the pages' routing format ("Stage 2: prior-induced sparse
 * softmax", implementation: the kernel iterates over the active chunks of a
 * bit-packed mask and adds the routing bias before the softmax).  The result
 * is that of dash_attn_sparse_ex on the lists holding the same blocks with
 * the same log p_bar values (bit-identical).  f16/bf16 only.
 *   mask     device uint32 [B, Hkv, S, n_words]: bit c % 32 of word c / 32 of
 *            a row set iff block c is selected for that query position (the
 *            layout dash_attn_lists_to_mask writes).  Bits on blocks that are
 *            not candidates of the row (its own block; later blocks when
 *            causal) are ignored and reported as DASH_ERR_INVALID_ARGUMENT in
 *            the workspace status word.
 *   n_words  words per row: n_words * 32 >= ceil(S / block), at most 128.
 *   logp     device fp32 [B, Hkv, S, t_cap]: log p_bar of block c at column c
 *            of the row; read only where the row's bit is set.
 *   workspace  dash_attn_sparse_workspace_size() bytes, 256-byte aligned.
 * Other arguments as for dash_attn_sparse_ex (opts: sigma only).
 */
dash_status_t dash_attn_sparse_mask(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                    const uint32_t* mask, int64_t n_words, const float* logp, int64_t t_cap, int block,
                                    int causal, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                    const dash_options_t* opts, dash_stream_t stream);

/*
 * dash_attn_decode without a workspace argument.  The paper has no
 * counterpart: this serves callers that may not allocate device memory
 * while they run -- code inside another engine's execution hook (a serving
 * runtime or graph-executor plugin) where allocation is forbidden or would
 * stall the device, and programs that fix their device-memory budget at
 * start-up.  The caller still passes inputs and outputs, exactly as for
 * dash_attn_decode, and gets the same results.
 *  - Scratch: one library-owned 16 MiB device array per GPU, held from the
 *    time the library is loaded until the process exits.  Problems whose
 *    dash_attn_decode_workspace_size() exceeds 16 MiB are refused with
 *    DASH_ERR_UNSUPPORTED before anything is launched.
 *  - The array is shared by all calls on a device and keeps the last call's
 *    contents; calls whose GPU work overlaps (other streams or threads
 *    without ordering) race and give wrong results.
 *  - The first call on each device looks up the array's address; make that
 *    first call before any stream capture.
 *  - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *  - The status word it uses is the array's: read it with
 *    dash_attn_decode_noalloc_status (a seqlens entry out of range is clamped
 *    and reported there as DASH_ERR_INVALID_ARGUMENT).
 *  - The address looked up by the first call stays valid for the life of the
 *    device's context; after cudaDeviceReset this entry point must not be
 *    called on that device again.
 */
dash_status_t dash_attn_decode_noalloc(const dash_tensor_t* q, const dash_tensor_t* kcache,
                                       const dash_tensor_t* vcache, const int32_t* seqlens, const float* summaries,
                                       int64_t t_cap, float alpha, int block, dash_tensor_t* out,
                                       dash_stream_t stream);

/*
 * Synchronises `stream`, then reads the status word of the last
 * dash_attn_decode_noalloc call on the current device (kept in its scratch
 * array), like dash_attn_get_device_status does for a workspace.  Returns
 * DASH_ERR_INVALID_ARGUMENT when no such call has been made on this device.
 * Allocates nothing.
 */
dash_status_t dash_attn_decode_noalloc_status(dash_stream_t stream);

/*
 * Test of the device-side timeout path (the paper has no counterpart): runs
 * the stage-2 tensor-core kernel of dash_attn_sparse on the same arguments,
 * but with its copy-issuing warp withholding every copy and every other wait
 * for a hand-off bounded by `wait_cycles` SM cycles (1024 .. 2^31) instead of
 * about a second.  Every such wait runs out; the kernel records
 * DASH_ERR_DEVICE_TIMEOUT in the workspace status word, frees its tensor
 * memory and returns, so the context stays usable and the next call on the
 * same workspace starts clean.  `out` is not written.  Nothing is left in
 * flight: waits that drain issued copies or MMAs keep the default bound.
 * f16/bf16 only.
 */
dash_status_t dash_attn_debug_sparse_stalled(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                             const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap,
                                             int block, int causal, dash_tensor_t* out, void* workspace,
                                             size_t workspace_bytes, int64_t wait_cycles, dash_stream_t stream);

/*
 * Synchronises `stream`, then reads the device status word of a workspace
 * last used by dash_attn_fwd / dash_attn_decode / dash_attn_sparse /
 * dash_attn_route / dash_attn_bwd (each call clears it when it starts).  Returns DASH_OK,
 * DASH_ERR_DEVICE_TIMEOUT (a bounded device wait expired; outputs of that
 * call are not valid), DASH_ERR_INVALID_ARGUMENT (a device-side value such
 * as seqlens[b] was out of range; it was clamped) or DASH_ERR_CUDA.
 */
dash_status_t dash_attn_get_device_status(void* workspace, dash_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DASHATTN_H_ */
