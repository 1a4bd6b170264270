// Stage 1 for prefill on the tensor cores: routing logits (tcgen05 GEMM kept
// in TMEM), alpha-entmax thresholds, GQA mean, per-row block lists and the
// stage-2 work lists of each tile.
//
// "Stage 1: entmax chunk routing" of the DashAttention technical summary:
// every query scores the chunk summaries, w = alpha-entmax(gamma z) gives a
// sparse distribution whose support size depends on the input, and under
// GQA the probabilities of the heads sharing a KV head are averaged into one
// shared sparse support.  gamma = 1/sqrt(d).
//
// One CTA owns the same 128-row tile as the stage-2 kernel (128 / G
// positions x G heads of one KV group).  Column c of the logit matrix is
// block c; a row masks the blocks that are not its candidates (causal: c >= t;
// otherwise its own block).
//   Logits: A = the query rows in fp32 (bf16/f16 values are exact in tf32),
//   B = the fp32 summaries split into a tf32 head and its exact fp32
//   remainder (also fed as tf32), two kind::tf32 MMAs accumulated in fp32:
//   about 21 significant bits of every summary reach the product, far below
//   the 1e-4 selection band.  128 rows x up to 512 columns fill TMEM.
//   Summaries stream through a double-buffered shared-memory stage that the
//   four row warps fill (splitting and swizzling on the way); one thread
//   issues the MMAs.
//   Thresholds: thread r owns row r (= TMEM lane r) and runs the same Newton
//   / exact-support solve as the CUDA-core routing kernel on its own row,
//   reading the logits from TMEM.
//   Output: per position, the blocks with p_bar > 0 in ascending order with
//   log p_bar (ballot/popc per 32 columns), and per tile the union of those
//   blocks plus the tile's own blocks, each with the mask of positions that
//   selected it, and the tile's number of 64-token steps.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace dash {
namespace {

constexpr int kRows = 128;
constexpr int kChunk = 64;          // candidates per B stage
constexpr int kMaxCols = 512;       // TMEM columns
constexpr int kWorkWarps = 16;      // loading, threshold and compaction warps
constexpr int kMmaWarp = kWorkWarps;
constexpr int kThreads = (kWorkWarps + 1) * 32;
constexpr int kWork = kWorkWarps * 32;
constexpr int kHalf = 64;           // rows whose logits sit in shared memory at once (512 columns)
constexpr int kXStride = kMaxCols + 4;  // widest row stride: 16-byte row starts, conflict-free 16-byte writes
constexpr int kSeed = 32;               // seed values per row: the top two of each 32-column chunk

struct RBars {
  uint64_t a_full;
  uint64_t b_full[2];
  uint64_t b_empty[2];
  uint64_t x_ready;
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct RLayout {
  static constexpr int KC = D / 32;                 // 128-byte chunks of an fp32 row
  static constexpr int kAChunk = kRows * 128;       // 16 KB
  static constexpr int kBChunk = kChunk * 128;      // 8 KB
  static constexpr int kBTerm = KC * kBChunk;       // one term of one stage
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + KC * kAChunk;  // [2 stages][hi, lo]
  static constexpr int kGemmBytes = kOffB + 2 * 2 * kBTerm;
  // logits of 64 wide or 128 narrow rows, over the GEMM operands (no longer needed then)
  static constexpr int kXBytes = (kGemmBytes > kHalf * kXStride * 4 ? kGemmBytes : kHalf * kXStride * 4);
  static constexpr int kOffMask = kXBytes;  // [512] uint4
  static constexpr int kOffList = kOffMask + kMaxCols * 16;  // per 32-column chunk: entries, steps [2][32]
  static constexpr int kOffSeed = kOffList + 2 * 32 * 4;  // [kRows][kSeed] fp32
  static constexpr int kOffBar = kOffSeed + kRows * kSeed * 4;
  static constexpr int kBytes = kOffBar + 128;
  static constexpr int kAlloc = kBytes + 1024;
};

// byte offset of 16-byte unit u of row r inside a 128-byte-swizzled chunk
__device__ __forceinline__ int sw128(int r, int u) { return r * 128 + ((u ^ (r & 7)) << 4); }

__device__ __forceinline__ float4 tf32_head(float4 v) {
  float4 h;
  h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
  h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
  h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
  h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
  return h;
}

// Warp-wide: every lane executes it with the same operands, one elected
// lane issues (see the warp-wide forms in tc.cuh).
__device__ __forceinline__ void mma_tf32_w(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Instruction descriptor, kind::tf32 (A/B format 2), fp32 accumulate, K-major.
constexpr uint32_t idesc_tf32(int m, int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Is logit column c a routing candidate of a row in block t?
__device__ __forceinline__ bool is_cand(int c, int t, int n_blocks, int causal) {
  return causal ? c < t : (c != t && c < n_blocks);
}

// Newton passes from below with the exact check on the current support, for
// RW rows in lockstep.  COLS = 1: each lane holds one value per row in v[i]
// (32 values per row); COLS = 2: row i's values are x[i * stride + c], read 64
// columns per iteration for c < n (readable, -inf, up to n rounded up to 64).
// tau[i] must be a lower bound of the root (F >= 1); rows with done[i] set are
// left alone.  KIND: 0 alpha = 2, 1 alpha = 1.5, 2 any other alpha.  The
// support size is summed and the smallest positive u taken over the warp
// with one redux each (u > 0, so its bits order as unsigned integers).
template <int RW, int COLS, int KIND>
__device__ __forceinline__ void entmax_newton_rows(const float* x, int stride, int n, float pw, int lane, float* tau,
                                                   bool* done) {
  for (int it = 0; it < 100; ++it) {
    float f[RW], a[RW], umin[RW], fd[RW];
    int k[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) f[i] = a[i] = fd[i] = 0.f, umin[i] = 3.0e38f, k[i] = 0;
    auto add = [&](int i, float xv) {
      const float u = xv - tau[i];
      if (u > 0.f) {
        k[i] += 1;
        a[i] += u;
        umin[i] = fminf(umin[i], u);
        if constexpr (KIND == 0) {
          f[i] += u;
        } else if constexpr (KIND == 1) {
          f[i] = fmaf(u, u, f[i]);
        } else {
          const float up = exp2f((pw - 1.0f) * log2f(u));
          fd[i] += up;
          f[i] = fmaf(up, u, f[i]);
        }
      }
    };
    if constexpr (COLS == 1) {
#pragma unroll
      for (int i = 0; i < RW; ++i) add(i, x[i]);
    } else {
      for (int c = lane; c < n; c += 64) {
        float xv[2 * RW];
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          xv[2 * i] = x[i * stride + c];
          xv[2 * i + 1] = x[i * stride + c + 32];
        }
#pragma unroll
        for (int e = 0; e < 2 * RW; ++e) add(e >> 1, xv[e]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        f[i] += __shfl_xor_sync(0xffffffffu, f[i], o);
        a[i] += __shfl_xor_sync(0xffffffffu, a[i], o);
        if constexpr (KIND == 2) fd[i] += __shfl_xor_sync(0xffffffffu, fd[i], o);
      }
    }
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      k[i] = (int)__reduce_add_sync(0xffffffffu, (unsigned)k[i]);
      umin[i] = __uint_as_float(__reduce_min_sync(0xffffffffu, __float_as_uint(umin[i])));
    }
    bool all = true;
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      if (!done[i]) {
        if constexpr (KIND == 0) {
          const float delta = (f[i] - 1.0f) / k[i];
          if (delta < umin[i]) {
            tau[i] += fmaxf(delta, 0.0f);
            done[i] = true;
          } else {
            tau[i] += delta;
          }
        } else if constexpr (KIND == 1) {
          const float disc = a[i] * a[i] - k[i] * (f[i] - 1.0f);
          float delta = 3.0e38f;
          if (disc >= 0.f) delta = (f[i] - 1.0f) / (a[i] + sqrtf(disc));
          if (delta < umin[i]) {
            tau[i] += fmaxf(delta, 0.0f);
            done[i] = true;
          } else {
            tau[i] += (f[i] - 1.0f) / (2.0f * a[i]);
          }
        } else {
          const float step = (f[i] - 1.0f) / (pw * fd[i]);
          tau[i] += step;
          if (fabsf(step) <= 1e-7f * fmaxf(1.0f, fabsf(tau[i]))) done[i] = true;
        }
      }
      all = all && done[i];
    }
    if (all) break;
  }
}

// alpha-entmax thresholds of RW rows that share their candidate columns,
// solved in lockstep by one warp.  Row i's logits are x[i * stride + c] for
// c < n, -inf on non-candidates, readable up to n rounded up to 64.  seed[i *
// kSeed + l] are kSeed values of row i (the top two of each 32-column chunk,
// -inf where a chunk has fewer): their maximum is the row's, and their
// threshold, solved first in registers, is a lower bound on the row's (F
// over the row >= F over any subset), so the passes over the row start there
// instead of at max - 1 and usually find the exact support at once.
template <int RW, int KIND>
__device__ __forceinline__ void warp_entmax_tau_rows(const float* x, int stride, int n, const float* seed,
                                                     float alpha, int lane, float* tau) {
  static_assert(kSeed == 32, "one seed value per lane");
  const float pw = 1.0f / (alpha - 1.0f);
  float sv[RW], mx[RW];
#pragma unroll
  for (int i = 0; i < RW; ++i) sv[i] = mx[i] = seed[i * kSeed + lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int i = 0; i < RW; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o));
  }
  bool done[RW];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    tau[i] = mx[i] - 1.0f;
    done[i] = mx[i] == kNegInf;
  }
  entmax_newton_rows<RW, 1, KIND>(sv, 0, 32, pw, lane, tau, done);
#pragma unroll
  for (int i = 0; i < RW; ++i) done[i] = mx[i] == kNegInf;
  entmax_newton_rows<RW, 2, KIND>(x, stride, n, pw, lane, tau, done);
}

// Thresholds, GQA mean and ascending per-position lists for the tile rows
// [row_base, row_base + round_rows), one warp per task of RW rows (RW / G
// positions x G heads) solved in lockstep.  Tile row r's logits (scaled,
// non-candidates -inf, readable up to the column count rounded up to 64) are
// X[(r - row_base) * xstride + c]; its seed values are
// seed[(r - row_base) * kSeed + l].  Marks in pmask[c] the tile positions
// that selected block c.  KIND is entmax_kind(p.alpha).
template <int G, int KIND>
__device__ __forceinline__ void solve_and_compact_k(const RouteParams& p, const float* X, int xstride,
                                                    const float* seed, uint4* pmask, int row_base, int round_rows,
                                                    int b, int g, int pos0, int n_blocks, int warp, int lane) {
  constexpr int RW = G > 4 ? G : 4;  // rows solved together by one warp
  constexpr int PPT = RW / G;        // positions per warp task
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const float pw = 1.0f / (p.alpha - 1.0f);
  const int n_tasks = round_rows / RW;
  for (int task = warp; task < n_tasks; task += kWorkWarps) {
    const int rr0 = task * RW;                 // first row within the round
    const int tp0 = (row_base + rr0) / G;      // first tile position
    const int pos = pos0 + tp0;
    const int t = pos / p.block;  // the task's positions share their block
    const int ncol = p.causal ? t : n_blocks;
    float tau[RW];
    // thresholds four rows at a time (register budget)
#pragma unroll
    for (int r4 = 0; r4 < RW; r4 += 4) {
      if (ncol > 0) {
        warp_entmax_tau_rows<4, KIND>(X + (rr0 + r4) * xstride, xstride, ncol, seed + (rr0 + r4) * kSeed, p.alpha,
                                      lane, tau + r4);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) tau[r4 + i] = 0.f;  // no candidates (nothing was copied)
      }
    }
#pragma unroll
    for (int pp = 0; pp < PPT; ++pp) {
      const int tp = tp0 + pp;
      const int qpos = pos0 + tp;
      if (qpos >= p.S) continue;
      const int n_row = p.causal ? t : n_blocks - 1;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (n_row == 0) tau[pp * G + h] = 0.f;
        if (p.tau && lane == 0) p.tau[((int64_t)b * p.H + g * G + h) * p.S + qpos] = tau[pp * G + h];
      }
      const int64_t row = bg * p.S + qpos;
      int32_t* idx = p.idx + row * p.t_cap;
      float* logp = p.logp + row * p.t_cap;
      int off = 0;
      for (int c0 = 0; c0 < ncol && n_row > 0; c0 += 32) {
        const int c = c0 + lane;
        float pbar = 0.f;
        if (c < ncol) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float u = X[(rr0 + pp * G + h) * xstride + c] - tau[pp * G + h];
            const float ph = u > 0.f ? pow_pw(u, pw, KIND) : 0.f;
            pbar += ph;
            if (p.p_dense) p.p_dense[(((int64_t)b * p.H + g * G + h) * p.S + qpos) * p.t_cap + c] = ph;
          }
          pbar *= 1.0f / (float)G;
        }
        const bool sel = pbar > 0.f;
        const unsigned m = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const int o = off + __popc(m & ((1u << lane) - 1u));
          idx[o] = c;
          logp[o] = logf(pbar);
          atomicOr(reinterpret_cast<uint32_t*>(&pmask[c]) + (tp >> 5), 1u << (tp & 31));
        }
        off += __popc(m);
      }
      if (lane == 0) p.cnt[row] = off;
      if (p.p_dense) {
        const int from = n_row > 0 ? ncol : 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float* pd = p.p_dense + (((int64_t)b * p.H + g * G + h) * p.S + qpos) * p.t_cap;
          for (int c = from + lane; c < p.t_cap; c += 32) pd[c] = 0.f;
        }
      }
    }
  }
}

template <int G>
__device__ __forceinline__ void solve_and_compact(const RouteParams& p, const float* X, int xstride, const float* seed,
                                                  uint4* pmask, int row_base, int round_rows, int b, int g, int pos0,
                                                  int n_blocks, int warp, int lane) {
  switch (entmax_kind(p.alpha)) {
    case 0:
      solve_and_compact_k<G, 0>(p, X, xstride, seed, pmask, row_base, round_rows, b, g, pos0, n_blocks, warp, lane);
      break;
    case 1:
      solve_and_compact_k<G, 1>(p, X, xstride, seed, pmask, row_base, round_rows, b, g, pos0, n_blocks, warp, lane);
      break;
    default:
      solve_and_compact_k<G, 2>(p, X, xstride, seed, pmask, row_base, round_rows, b, g, pos0, n_blocks, warp, lane);
  }
}

// The tile's stage-2 work list: the union of its positions' blocks plus the
// tile's own blocks, ascending, each with the mask of positions that
// selected it, and the tile's number of 64-token steps.  One warp per
// 32-column chunk counts, then every chunk writes at its prefix offset.
// pmask[c] (c < pmask_cap) holds the positions that selected block c; lcnt
// and lsteps have one entry per 32-column chunk.  Called by every thread of
// the CTA (it contains a CTA barrier).
__device__ __forceinline__ void write_tile_list(const RouteParams& p, const TileOut& to, const uint4* pmask,
                                                int pmask_cap, int* lcnt, int* lsteps, int64_t bg, int tile, int pos0,
                                                int last, int t_last, int n_cols, int warp, int lane) {
  const int own_lo = pos0 / p.block, own_hi = t_last;
  const int last_needed = p.causal ? last : p.S - 1;
  const int span = max(n_cols, own_hi + 1);
  const int n_lch = (span + 31) / 32;
  auto chunk = [&](int ch, uint4& m, unsigned& bal, int& st) {
    const int c = ch * 32 + lane;
    bool keep = false;
    m = make_uint4(0u, 0u, 0u, 0u);
    st = 0;
    if (c < span) {
      if (c < pmask_cap) m = pmask[c];
      keep = (m.x | m.y | m.z | m.w) != 0u || (c >= own_lo && c <= own_hi);
      if (keep)
        for (int h = 0; h < p.block / 64; ++h) st += (c * p.block + h * 64 <= last_needed) ? 1 : 0;
    }
    bal = __ballot_sync(0xffffffffu, keep);
    return keep;
  };
  if (warp < kWorkWarps) {
    for (int ch = warp; ch < n_lch; ch += kWorkWarps) {
      uint4 m;
      unsigned bal;
      int st;
      chunk(ch, m, bal, st);
      st = warp_sum_i(st);
      if (lane == 0) {
        lcnt[ch] = __popc(bal);
        lsteps[ch] = st;
      }
    }
  }
  __syncthreads();
  if (warp < kWorkWarps) {
    const int64_t tix = bg * to.n_tiles + tile;
    int32_t* out = to.ulist + tix * p.t_cap;
    uint4* mout = to.umask + tix * p.t_cap;
    for (int ch = warp; ch < n_lch; ch += kWorkWarps) {
      uint4 m;
      unsigned bal;
      int st;
      const bool keep = chunk(ch, m, bal, st);
      int off = 0;
      for (int k = 0; k < ch; ++k) off += lcnt[k];
      if (keep) {
        const int k = off + __popc(bal & ((1u << lane) - 1u));
        out[k] = ch * 32 + lane;
        mout[k] = m;
      }
    }
    if (warp == 0) {
      int n = 0, steps = 0;
      for (int k = lane; k < n_lch; k += 32) {
        n += lcnt[k];
        steps += lsteps[k];
      }
      n = warp_sum_i(n);
      steps = warp_sum_i(steps);
      if (lane == 0) {
        to.ucnt[tix] = n;
        to.usteps[tix] = steps;
      }
    }
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) route_prefill_tc_kernel(RouteParams p, TileOut to, int tile0) {
  using L = RLayout<D>;
  constexpr uint32_t kIdesc = idesc_tf32(kRows, kChunk);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RBars* bars = reinterpret_cast<RBars*>(smem + L::kOffBar);
  float* X = reinterpret_cast<float*>(smem);  // [round rows][xstride], after the GEMM
  float* seed = reinterpret_cast<float*>(smem + L::kOffSeed);  // [round rows][kSeed]
  uint4* pmask = reinterpret_cast<uint4*>(smem + L::kOffMask);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y, tile = tile0 + blockIdx.x;
  constexpr int P = kRows / G;
  const int pos0 = tile * P;
  const int n_blocks = (p.S + p.block - 1) / p.block;
  const int last = min(pos0 + P, p.S) - 1;
  const int t_last = last / p.block;
  const int n_cols = p.causal ? t_last : n_blocks;  // logit columns 0 .. n_cols-1
  const int n_chunks = (n_cols + kChunk - 1) / kChunk;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const float coef = (p.alpha - 1.0f) * rsqrtf((float)D);

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->a_full, kWork);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->b_full[s], p.summ_split ? 1 : kWork);
      tc::mbar_init(&bars->b_empty[s], 1);
    }
    tc::mbar_init(&bars->x_ready, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  for (int c = threadIdx.x; c < kMaxCols; c += kThreads) pmask[c] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&bars->tmem_base, kMaxCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // whole warp (uniform descriptors), one elected lane issues
    if (n_chunks > 0) {
      bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->a_full, 0));
      const uint64_t adesc0 = tc::smem_desc_sw128(smem + L::kOffA, 16, 1024);
      const uint64_t bdesc0 = tc::smem_desc_sw128(smem + L::kOffB, 16, 1024);
      for (int j = 0; ok && j < n_chunks; ++j) {
        const int st = j & 1;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->b_full[st], (j >> 1) & 1))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int term = 0; term < 2; ++term) {
          const uint64_t bd = bdesc0 + (uint64_t)(((st * 2 + term) * L::kBTerm) >> 4);
#pragma unroll
          for (int kc = 0; kc < L::KC; ++kc) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_tf32_w(tmem + j * kChunk, adesc0 + (uint64_t)((kc * L::kAChunk + k * 32) >> 4),
                         bd + (uint64_t)((kc * L::kBChunk + k * 32) >> 4), kIdesc, (term | kc | k) ? 1u : 0u);
          }
        }
        tc::mma_commit_w(&bars->b_empty[st]);
      }
      if (!ok) {
        raise_status(p.status, 5 /* DASH_ERR_DEVICE_TIMEOUT */, 20);
        atomicExch(&bars->abort, 1);
      }
      tc::mma_commit_w(&bars->x_ready);
      tc::mbar_wait(&bars->x_ready, 0);
    }
  } else if (n_chunks > 0) {
    // ------------------------------------------------------------ GEMM operands
    bool ok = true;
    if (threadIdx.x < kRows) {
      // A: query row r in fp32, 128-byte swizzled
      const int r = threadIdx.x;
      const int pos = pos0 + r / G, head = g * G + r % G;
      const bool valid = pos < p.S;
      constexpr int EPV = 8;
      const T* src = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)(valid ? pos : 0) * p.q.ss +
                     (int64_t)head * p.q.sh;
#pragma unroll
      for (int v = 0; v < D / EPV; ++v) {
        float f[EPV];
        if (valid) {
          Elt<T>::to_float(__ldg(reinterpret_cast<const uint4*>(src + v * EPV)), f);
        } else {
#pragma unroll
          for (int e = 0; e < EPV; ++e) f[e] = 0.f;
        }
        const int kc = (v * EPV) / 32, u0 = ((v * EPV) % 32) / 4;
        uint8_t* base = smem + L::kOffA + kc * L::kAChunk;
        *reinterpret_cast<float4*>(base + sw128(r, u0)) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(base + sw128(r, u0 + 1)) = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars->a_full);
    if (p.summ_split) {
      // B: the pre-split chunks, two bulk copies per stage by one thread
      if (warp == kWorkWarps - 1 && lane == 0) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.summ_split) +
                             bg * (int64_t)((p.t_cap + kChunk - 1) / kChunk) * 2 * L::kBTerm;
        for (int j = 0; j < n_chunks; ++j) {
          const int st = j & 1;
          if (j >= 2 && !tc::mbar_wait(&bars->b_empty[st], ((j >> 1) - 1) & 1)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&bars->b_full[st], 2 * L::kBTerm);
          tc::bulk_load(smem + L::kOffB + (st * 2) * L::kBTerm, src + (int64_t)j * 2 * L::kBTerm, 2 * L::kBTerm,
                        &bars->b_full[st]);
        }
      }
    } else {
      // B: summaries of each candidate chunk, split into tf32 head + remainder.
      // The loads of chunk j + 1 are issued before chunk j is stored, so their
      // latency overlaps the wait for a free stage and the stores.
      const float* sbase = p.summaries + bg * p.t_cap * D;
      constexpr int EPT = kChunk * (D / 4) / kWork;  // float4 per thread and chunk
      static_assert(EPT * kWork == kChunk * (D / 4), "chunk not divisible among the loading threads");
      auto load_chunk = [&](int j, float4* v) {
  #pragma unroll
        for (int e = 0; e < EPT; ++e) {
          const int i = threadIdx.x + e * kWork;
          const int cand = i / (D / 4), k4 = i % (D / 4);
          const int c = j * kChunk + cand;
          v[e] = c < n_cols ? __ldg(reinterpret_cast<const float4*>(sbase + (int64_t)c * D) + k4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      };
      float4 cur[EPT], nxt[EPT];
      load_chunk(0, cur);
      for (int j = 0; j < n_chunks; ++j) {
        const int st = j & 1;
        if (j + 1 < n_chunks) load_chunk(j + 1, nxt);
        if (j >= 2 && !tc::mbar_wait(&bars->b_empty[st], ((j >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* bh = smem + L::kOffB + (st * 2 + 0) * L::kBTerm;
        uint8_t* bl = smem + L::kOffB + (st * 2 + 1) * L::kBTerm;
  #pragma unroll
        for (int e = 0; e < EPT; ++e) {
          const int i = threadIdx.x + e * kWork;
          const int cand = i / (D / 4), k4 = i % (D / 4);
          const float4 v = cur[e];
          const float4 h = tf32_head(v);
          const float4 lo = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
          const int kc = k4 / 8, u = k4 % 8;
          *reinterpret_cast<float4*>(bh + kc * L::kBChunk + sw128(cand, u)) = h;
          *reinterpret_cast<float4*>(bl + kc * L::kBChunk + sw128(cand, u)) = lo;
          cur[e] = nxt[e];
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bars->b_full[st]);
      }
    }
    if (ok && !tc::mbar_wait(&bars->x_ready, 0)) ok = false;
    tc::fence_after_sync();
    if (!ok) {
      raise_status(p.status, 5 /* DASH_ERR_DEVICE_TIMEOUT */, 21);
      atomicExch(&bars->abort, 1);
    }
  }
  __syncthreads();  // GEMM done: its shared memory now holds logits

  // ---- rounds of rows: TMEM -> shared, thresholds, compaction.  All 128
  // rows in one round when their logits fit the buffer (up to 256 columns),
  // else two rounds of 64.
  // 32-column chunks of the logit rows, an even number: the threshold passes
  // read columns in pairs of chunks (the extra columns hold -inf)
  const int n_wch = ((n_cols + 63) / 64) * 2;
  const int xstride = n_wch * 32 + 4;
  const int round_rows = kRows * xstride * 4 <= L::kXBytes ? kRows : kHalf;
  for (int half = 0; half * round_rows < kRows; ++half) {
    if (warp < kWorkWarps && n_chunks > 0 && !bars->abort) {
      // warps whose TMEM lane quarter lies in this round copy (and scale) their rows
      const int q4 = warp & 3;
      if (q4 * 32 >= half * round_rows && q4 * 32 < (half + 1) * round_rows) {
        const int r = q4 * 32 + lane;  // tile row = TMEM lane
        const int pos = pos0 + r / G;
        const int t = pos / p.block;
        const bool valid = pos < p.S;
        float* xr = X + (r - half * round_rows) * xstride;
        float* sr = seed + (r - half * round_rows) * kSeed;
        for (int ch = warp >> 2; ch < n_wch; ch += kWorkWarps / 4) {
          uint32_t v[32];
          tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + ch * 32, v);
          tc::tmem_wait_ld();
          float m1 = kNegInf, m2 = kNegInf;  // top two of the chunk
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = ch * 32 + j + e;
              y[e] = (valid && is_cand(c, t, n_blocks, p.causal)) ? coef * __uint_as_float(v[j + e]) : kNegInf;
              m2 = fmaxf(m2, fminf(m1, y[e]));
              m1 = fmaxf(m1, y[e]);
            }
            *reinterpret_cast<float4*>(xr + ch * 32 + j) = make_float4(y[0], y[1], y[2], y[3]);
          }
          sr[2 * ch] = m1;
          sr[2 * ch + 1] = m2;
        }
        for (int e = 2 * n_wch + (warp >> 2); e < kSeed; e += kWorkWarps / 4) sr[e] = kNegInf;
      }
    }
    __syncthreads();
    if (warp < kWorkWarps)
      solve_and_compact<G>(p, X, xstride, seed, pmask, half * round_rows, round_rows, b, g, pos0, n_blocks, warp, lane);
    __syncthreads();
  }

  // ---- the tile's stage-2 work list: the union of the positions' blocks
  // plus the tile's own blocks, ascending; one warp per 32-column chunk
  // counts, then every chunk writes at its prefix offset
  tc::fence_before_sync();
  if (to.ulist) {
    int* lcnt = reinterpret_cast<int*>(smem + L::kOffList);
    write_tile_list(p, to, pmask, kMaxCols, lcnt, lcnt + 32, bg, tile, pos0, last, t_last, n_cols, warp, lane);
  }
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kMaxCols);
  }
}

// ---------------------------------------------------------------------------
// Tiles with more candidate columns than TMEM holds (long contexts, up to
// 4096 blocks).  The logits are computed in segments of 512 columns; after
// each segment the work warps move it from TMEM into this CTA's scratch slot
// in global memory (128 rows x the tile's columns in fp32, at most 2 MB; the
// slots of the CTAs in flight stay in L2), scaled and masked as above, and
// keep one seed value per row and 32-column chunk slot (the running maximum
// of the chunks that map to it: still a subset of the row, so its threshold
// is still a lower bound).  Thresholds, lists and the tile's work list are
// then solved over the slot by the same code as the narrow kernel.  A CTA
// claims a free slot with a compare-and-swap on its lock word (there are
// more slots than CTAs of this kernel can be resident, one per SM) and frees
// it before it exits.

constexpr int kWideMaxCols = 4096;
constexpr int kSegChunks = kMaxCols / kChunk;  // GEMM chunks per 512-column segment
constexpr int kWideListCap = kWideMaxCols / 32 + 8;
constexpr int kOffWideList = kWideMaxCols * 16;  // after the [4096] uint4 position masks

struct WBars {
  uint64_t a_full;
  uint64_t b_full[2];
  uint64_t b_empty[2];
  uint64_t x_ready;    // one phase per segment: its MMAs are complete
  uint64_t tmem_free;  // one phase per segment: every work warp has read it
  uint64_t drain;      // every MMA issued is complete
  uint32_t tmem_base;
  int abort;
  int slot;
};
static_assert(sizeof(WBars) <= 128, "barriers must fit the reserved bytes");

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    route_prefill_tc_wide_kernel(RouteParams p, TileOut to, int tile0, WideScratch wsc) {
  using L = RLayout<D>;
  static_assert(kOffWideList + 2 * kWideListCap * 4 <= L::kGemmBytes, "wide-tile lists must fit over the operands");
  constexpr uint32_t kIdesc = idesc_tf32(kRows, kChunk);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WBars* bars = reinterpret_cast<WBars*>(smem + L::kOffBar);
  float* seed = reinterpret_cast<float*>(smem + L::kOffSeed);  // [kRows][kSeed]
  uint4* pmask = reinterpret_cast<uint4*>(smem);               // over the operands, once the GEMMs are done
  int* lcnt = reinterpret_cast<int*>(smem + kOffWideList);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y, tile = tile0 + blockIdx.x;
  constexpr int P = kRows / G;
  const int pos0 = tile * P;
  const int n_blocks = (p.S + p.block - 1) / p.block;
  const int last = min(pos0 + P, p.S) - 1;
  const int t_last = last / p.block;
  const int n_cols = p.causal ? t_last : n_blocks;
  const int n_chunks = (n_cols + kChunk - 1) / kChunk;
  const int n_seg = (n_chunks + kSegChunks - 1) / kSegChunks;
  const int n_wch = 2 * n_chunks;  // 32-column chunks, an even number
  const int xstride = n_wch * 32 + 4;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const float coef = (p.alpha - 1.0f) * rsqrtf((float)D);

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->a_full, kWork);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->b_full[s], 1);
      tc::mbar_init(&bars->b_empty[s], 1);
    }
    tc::mbar_init(&bars->x_ready, 1);
    tc::mbar_init(&bars->tmem_free, kWorkWarps);
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
    // There are more slots than CTAs of this kernel can be resident, so one
    // is free; sweeps repeat (bounded) because the release of the CTA this one
    // replaces may still be on its way to memory.
    int slot = -1;
    const int64_t cta = blockIdx.x + (int64_t)gridDim.x * (blockIdx.y + (int64_t)gridDim.y * blockIdx.z);
    const int start = (int)(cta % wsc.n_slots);
    const long long t0 = clock64();
    for (int sweep = 0; slot < 0; ++sweep) {
      for (int i = 0; i < wsc.n_slots && slot < 0; ++i) {
        const int s = (start + i) % wsc.n_slots;
        if (atomicCAS(&wsc.locks[s], 0, 1) == 0) slot = s;
      }
      if (slot < 0 && clock64() - t0 > (1ll << 26)) break;
    }
    bars->slot = slot;
    if (slot < 0) raise_status(p.status, 4 /* DASH_ERR_CUDA */, 23);
  }
  for (int i = threadIdx.x; i < kRows * kSeed; i += kThreads) seed[i] = kNegInf;
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&bars->tmem_base, kMaxCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const int slot = bars->slot;
  const bool live = slot >= 0 && n_chunks > 0;
  float* X = live ? wsc.logits + (int64_t)slot * wsc.slot_floats : nullptr;

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (live) {
      bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->a_full, 0));
      const uint64_t adesc0 = tc::smem_desc_sw128(smem + L::kOffA, 16, 1024);
      const uint64_t bdesc0 = tc::smem_desc_sw128(smem + L::kOffB, 16, 1024);
      for (int s = 0; ok && s < n_seg; ++s) {
        if (s > 0) {
          // the work warps have moved the previous segment out of TMEM
          if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->tmem_free, (s - 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
        const int j_end = min(n_chunks, (s + 1) * kSegChunks);
        for (int j = s * kSegChunks; j < j_end; ++j) {
          const int st = j & 1;
          if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->b_full[st], (j >> 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
#pragma unroll
          for (int term = 0; term < 2; ++term) {
            const uint64_t bd = bdesc0 + (uint64_t)(((st * 2 + term) * L::kBTerm) >> 4);
#pragma unroll
            for (int kc = 0; kc < L::KC; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_tf32_w(tmem + (j - s * kSegChunks) * kChunk,
                           adesc0 + (uint64_t)((kc * L::kAChunk + k * 32) >> 4),
                           bd + (uint64_t)((kc * L::kBChunk + k * 32) >> 4), kIdesc, (term | kc | k) ? 1u : 0u);
            }
          }
          tc::mma_commit_w(&bars->b_empty[st]);
        }
        if (!ok) break;
        tc::mma_commit_w(&bars->x_ready);
      }
      if (!ok) {
        raise_status(p.status, 5 /* DASH_ERR_DEVICE_TIMEOUT */, 24);
        atomicExch(&bars->abort, 1);
      }
      tc::mma_commit_w(&bars->drain);
      tc::mbar_wait(&bars->drain, 0);
    }
  } else if (live) {
    // ------------------------------------------------------------ operands and segment copies
    if (threadIdx.x < kRows) {
      // A: query row r in fp32, 128-byte swizzled
      const int r = threadIdx.x;
      const int pos = pos0 + r / G, head = g * G + r % G;
      const bool valid = pos < p.S;
      constexpr int EPV = 8;
      const T* src = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)(valid ? pos : 0) * p.q.ss +
                     (int64_t)head * p.q.sh;
#pragma unroll
      for (int v = 0; v < D / EPV; ++v) {
        float f[EPV];
        if (valid) {
          Elt<T>::to_float(__ldg(reinterpret_cast<const uint4*>(src + v * EPV)), f);
        } else {
#pragma unroll
          for (int e = 0; e < EPV; ++e) f[e] = 0.f;
        }
        const int kc = (v * EPV) / 32, u0 = ((v * EPV) % 32) / 4;
        uint8_t* base = smem + L::kOffA + kc * L::kAChunk;
        *reinterpret_cast<float4*>(base + sw128(r, u0)) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(base + sw128(r, u0 + 1)) = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars->a_full);

    const bool loader = warp == kWorkWarps - 1 && lane == 0;
    const uint8_t* split = reinterpret_cast<const uint8_t*>(p.summ_split) +
                           bg * (int64_t)((p.t_cap + kChunk - 1) / kChunk) * 2 * L::kBTerm;
    int issued = 0;
    bool lok = true;
    bool ok = true;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // tile row = TMEM lane
    const int pos = pos0 + r / G;
    const int t = pos / p.block;
    const bool valid = pos < p.S;
    float* xr = X + (int64_t)r * xstride;
    float* sr = seed + r * kSeed;
    for (int s = 0; s < n_seg; ++s) {
      if (loader) {
        // this segment's chunks and the first two of the next (their stages
        // free up without waiting for this segment's copy)
        const int j_end = min(n_chunks, (s + 1) * kSegChunks + 2);
        for (; lok && issued < j_end; ++issued) {
          const int j = issued, st = j & 1;
          if (j >= 2 && !tc::mbar_wait(&bars->b_empty[st], ((j >> 1) - 1) & 1)) {
            lok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&bars->b_full[st], 2 * L::kBTerm);
          tc::bulk_load(smem + L::kOffB + (st * 2) * L::kBTerm, split + (int64_t)j * 2 * L::kBTerm, 2 * L::kBTerm,
                        &bars->b_full[st]);
        }
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->x_ready, s & 1));
      if (!ok) break;
      tc::fence_after_sync();
      const int ch0 = s * (kMaxCols / 32), ch1 = min(n_wch, ch0 + kMaxCols / 32);
      for (int ch = ch0 + (warp >> 2); ch < ch1; ch += kWorkWarps / 4) {
        uint32_t v[32];
        tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + (ch - ch0) * 32, v);
        tc::tmem_wait_ld();
        float m1 = kNegInf;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = ch * 32 + j + e;
            y[e] = (valid && is_cand(c, t, n_blocks, p.causal)) ? coef * __uint_as_float(v[j + e]) : kNegInf;
            m1 = fmaxf(m1, y[e]);
          }
          *reinterpret_cast<float4*>(xr + ch * 32 + j) = make_float4(y[0], y[1], y[2], y[3]);
        }
        sr[ch & 31] = fmaxf(sr[ch & 31], m1);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->tmem_free);
    }
    if (!ok) {
      raise_status(p.status, 5 /* DASH_ERR_DEVICE_TIMEOUT */, 25);
      atomicExch(&bars->abort, 1);
    }
    if (loader) {
      // no bulk copy may still be landing in shared memory past this point
      for (int j = max(0, issued - 2); j < issued; ++j) tc::mbar_wait(&bars->b_full[j & 1], (j >> 1) & 1);
    }
  }
  __syncthreads();  // segments done: the slot holds the logits, the operand memory is free

  const bool run = live && bars->abort == 0;
  if (run)
    for (int c = threadIdx.x; c < n_wch * 32; c += kThreads) pmask[c] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (run && warp < kWorkWarps)
    solve_and_compact<G>(p, X, xstride, seed, pmask, 0, kRows, b, g, pos0, n_blocks, warp, lane);
  __syncthreads();
  if (threadIdx.x == 0 && slot >= 0) {
    __threadfence();  // this CTA's reads of the slot are done before another CTA may claim it
    atomicExch(&wsc.locks[slot], 0);
  }
  if (run && to.ulist)
    write_tile_list(p, to, pmask, n_wch * 32, lcnt, lcnt + kWideListCap, bg, tile, pos0, last, t_last, n_cols,
                    warp, lane);
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kMaxCols);
  }
}

template <typename T, int D, int G>
cudaError_t launch_wide_g(const RouteParams& p, const TileOut& to, int tile0, int n_tiles, const WideScratch& w,
                          cudaStream_t stream) {
  using L = RLayout<D>;
  auto kern = route_prefill_tc_wide_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles, p.Hkv, p.B);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p, to, tile0, w);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_wide_t(const RouteParams& p, const TileOut& to, int tile0, int n_tiles, const WideScratch& w,
                          cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_wide_g<T, D, 1>(p, to, tile0, n_tiles, w, stream);
    case 2: return launch_wide_g<T, D, 2>(p, to, tile0, n_tiles, w, stream);
    case 4: return launch_wide_g<T, D, 4>(p, to, tile0, n_tiles, w, stream);
    default: return launch_wide_g<T, D, 8>(p, to, tile0, n_tiles, w, stream);
  }
}

template <typename T, int D, int G>
cudaError_t launch_g(const RouteParams& p, const TileOut& to, int tile0, int n_tiles, cudaStream_t stream) {
  using L = RLayout<D>;
  auto kern = route_prefill_tc_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles, p.Hkv, p.B);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p, to, tile0);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_t(const RouteParams& p, const TileOut& to, int tile0, int n_tiles, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_g<T, D, 1>(p, to, tile0, n_tiles, stream);
    case 2: return launch_g<T, D, 2>(p, to, tile0, n_tiles, stream);
    case 4: return launch_g<T, D, 4>(p, to, tile0, n_tiles, stream);
    default: return launch_g<T, D, 8>(p, to, tile0, n_tiles, stream);
  }
}

// The summaries of one (batch, KV head) chunk of 64 candidates, split into
// the tf32 head and its remainder and laid out exactly as the routing
// kernel's B stage (128-byte swizzled K-major chunks, head then remainder),
// zero past t_cap.
template <int D>
__global__ void __launch_bounds__(256) route_split_kernel(const float* summaries, int64_t t_cap, float* split) {
  using L = RLayout<D>;
  const int j = blockIdx.x;
  const int64_t bg = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int64_t n_ch = (t_cap + kChunk - 1) / kChunk;
  uint8_t* dst = reinterpret_cast<uint8_t*>(split) + (bg * n_ch + j) * 2 * L::kBTerm;
  const float* sbase = summaries + bg * t_cap * D;
  for (int i = threadIdx.x; i < kChunk * (D / 4); i += blockDim.x) {
    const int cand = i / (D / 4), k4 = i % (D / 4);
    const int64_t c = (int64_t)j * kChunk + cand;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c < t_cap) v = __ldg(reinterpret_cast<const float4*>(sbase + c * D) + k4);
    const float4 h = tf32_head(v);
    const int kc = k4 / 8, u = k4 % 8;
    *reinterpret_cast<float4*>(dst + kc * L::kBChunk + sw128(cand, u)) = h;
    *reinterpret_cast<float4*>(dst + L::kBTerm + kc * L::kBChunk + sw128(cand, u)) =
        make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
  }
}

}  // namespace

int route_tc_max_cols() { return kMaxCols; }

int route_tc_wide_max_cols() { return kWideMaxCols; }

size_t route_wide_scratch_bytes(int64_t t_cap, int n_slots) {
  const int64_t slot_floats = (int64_t)kRows * (((t_cap + 63) / 64) * 64 + 4);
  const size_t locks = ((size_t)n_slots * 4 + 255) & ~size_t(255);
  return locks + (size_t)n_slots * (size_t)slot_floats * 4;
}

WideScratch route_wide_scratch(void* base, int64_t t_cap, int n_slots) {
  WideScratch w{};
  const size_t locks = ((size_t)n_slots * 4 + 255) & ~size_t(255);
  w.locks = static_cast<int32_t*>(base);
  w.logits = reinterpret_cast<float*>(static_cast<char*>(base) + locks);
  w.n_slots = n_slots;
  w.slot_floats = (int64_t)kRows * (((t_cap + 63) / 64) * 64 + 4);
  return w;
}

cudaError_t launch_route_prefill_tc_wide(const RouteParams& p, const TileOut& to, int tile0, int n_tiles,
                                         const WideScratch& w, cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  if (!p.summ_split || !w.locks || w.n_slots <= 0) return cudaErrorInvalidValue;
  if (p.D == 128) {
    if (p.dtype == 1) return launch_wide_t<__half, 128>(p, to, tile0, n_tiles, w, stream);
    return launch_wide_t<__nv_bfloat16, 128>(p, to, tile0, n_tiles, w, stream);
  }
  if (p.dtype == 1) return launch_wide_t<__half, 64>(p, to, tile0, n_tiles, w, stream);
  return launch_wide_t<__nv_bfloat16, 64>(p, to, tile0, n_tiles, w, stream);
}

size_t route_split_bytes(int64_t B, int64_t Hkv, int64_t t_cap, int D) {
  return (size_t)(B * Hkv) * (size_t)((t_cap + kChunk - 1) / kChunk) * 2 * (size_t)(D / 32) * kChunk * 128;
}

cudaError_t launch_route_split(const RouteParams& p, float* split, cudaStream_t stream) {
  dim3 grid((unsigned)((p.t_cap + kChunk - 1) / kChunk), p.Hkv, p.B);
  if (p.D == 128)
    route_split_kernel<128><<<grid, 256, 0, stream>>>(p.summaries, p.t_cap, split);
  else
    route_split_kernel<64><<<grid, 256, 0, stream>>>(p.summaries, p.t_cap, split);
  return cudaGetLastError();
}

cudaError_t launch_route_prefill_tc(const RouteParams& p, const TileOut& to, int tile0, int n_tiles,
                                    cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  if (p.D == 128) {
    if (p.dtype == 1) return launch_t<__half, 128>(p, to, tile0, n_tiles, stream);
    return launch_t<__nv_bfloat16, 128>(p, to, tile0, n_tiles, stream);
  }
  if (p.dtype == 1) return launch_t<__half, 64>(p, to, tile0, n_tiles, stream);
  return launch_t<__nv_bfloat16, 64>(p, to, tile0, n_tiles, stream);
}

}  // namespace dash
