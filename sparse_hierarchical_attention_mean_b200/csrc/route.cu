// Stage 1 for prefill: routing scores, alpha-entmax, GQA average and the
// compaction of each query row's support into an ascending block list.
//
// "Stage 1: entmax chunk routing" of the DashAttention technical summary:
// each query scores the chunk summaries, w = alpha-entmax(gamma z) gives a
// sparse distribution whose support size depends on the input, and under
// GQA the probabilities of the query heads sharing a KV head are averaged
// into one shared sparse support.  gamma = 1/sqrt(d).
//
// One CTA owns R rows = (R / G positions) x (G heads of one KV group); all
// positions of a CTA lie in one block, so they share the N candidates.  The
// CTA computes the R x N logits into shared memory chunk by chunk (fp32
// CUDA-core GEMM, summaries staged with cp.async), solves tau for every row
// with one warp per row, then one warp per position averages the G heads
// and writes the list with a ballot/popc scan.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int cand_block(int ci, int t, int causal) {
  return causal ? ci : (ci < t ? ci : ci + 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) route_prefill_kernel(RouteParams p, int R, int CW) {
  extern __shared__ __align__(16) float smem[];
  constexpr int DP = D + 4;
  __shared__ float tau_s[64];

  const int b = blockIdx.z, g = blockIdx.y;
  const int G = p.G;
  const int rpos = R / G;
  const int pos0 = p.pos_begin + blockIdx.x * rpos;
  const int t = pos0 / p.block;
  const int T_ = (p.S + p.block - 1) / p.block;
  const int N = p.causal ? t : T_ - 1;
  const int NP = (N + 3) & ~3;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float pw = 1.0f / (p.alpha - 1.0f);
  const int kind = entmax_kind(p.alpha);
  const int64_t bg = (int64_t)b * p.Hkv + g;

  float* Qs = smem;           // [R][DP]
  float* Ss = Qs + R * DP;    // [CW][DP]
  float* X = Ss + CW * DP;    // [R][NP]

  if (N > 0) {
    // ---- query rows -> fp32 shared memory
    constexpr int EPV = Elt<T>::kPerVec;
    constexpr int VPR = D / EPV;
    for (int i = tid; i < R * VPR; i += kThreads) {
      const int r = i / VPR, v = i % VPR;
      const int pos = pos0 + r / G, head = g * G + r % G;
      float f[EPV];
      if (pos < p.S) {
        const T* src = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)pos * p.q.ss +
                       (int64_t)head * p.q.sh + v * EPV;
        Elt<T>::to_float(__ldg(reinterpret_cast<const uint4*>(src)), f);
      } else {
#pragma unroll
        for (int e = 0; e < EPV; ++e) f[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < EPV; ++e) Qs[r * DP + v * EPV + e] = f[e];
    }

    // ---- logits x = (alpha - 1) / sqrt(d) * q . s_c
    const float coef = (p.alpha - 1.0f) * rsqrtf((float)D);
    const float* sbase = p.summaries + bg * p.t_cap * D;
    const int cq = CW / 4;
    const int rg = tid / cq, cg = tid % cq;
    for (int ch0 = 0; ch0 < N; ch0 += CW) {
      for (int i = tid; i < CW * (D / 4); i += kThreads) {
        const int cand = i / (D / 4), k4 = i % (D / 4);
        const int ci = ch0 + cand;
        const bool ok = ci < N;
        const float* src = sbase + (int64_t)(ok ? cand_block(ci, t, p.causal) : 0) * D + 4 * k4;
        cp_async16(Ss + cand * DP + 4 * k4, src, ok);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      if (rg < R / 4) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
        for (int k4 = 0; k4 < D / 4; ++k4) {
          float4 qv[4], sv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) qv[i] = *reinterpret_cast<const float4*>(Qs + (4 * rg + i) * DP + 4 * k4);
#pragma unroll
          for (int j = 0; j < 4; ++j) sv[j] = *reinterpret_cast<const float4*>(Ss + (cg + cq * j) * DP + 4 * k4);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              acc[i][j] = fmaf(qv[i].x, sv[j].x, acc[i][j]);
              acc[i][j] = fmaf(qv[i].y, sv[j].y, acc[i][j]);
              acc[i][j] = fmaf(qv[i].z, sv[j].z, acc[i][j]);
              acc[i][j] = fmaf(qv[i].w, sv[j].w, acc[i][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = ch0 + cg + cq * j;
          if (c < NP) {
#pragma unroll
            for (int i = 0; i < 4; ++i) X[(4 * rg + i) * NP + c] = coef * acc[i][j];
          }
        }
      }
      __syncthreads();
    }

    // ---- tau per row (one warp per row)
    for (int r = warp; r < R; r += kThreads / 32) {
      const int pos = pos0 + r / G;
      float tau = 0.f;
      if (pos < p.S) tau = warp_entmax_tau(X + r * NP, N, p.alpha, lane);
      if (lane == 0) tau_s[r] = tau;
    }
    __syncthreads();
  }

  // ---- GQA average + compaction (one warp per position)
  for (int pp = warp; pp < rpos; pp += kThreads / 32) {
    const int pos = pos0 + pp;
    if (pos >= p.S) continue;
    const int64_t row = (bg * p.S + pos);
    int32_t* idx = p.idx + row * p.t_cap;
    float* logp = p.logp + row * p.t_cap;
    int off = 0;
    for (int c0 = 0; c0 < N; c0 += 32) {
      const int c = c0 + lane;
      float pb = 0.f;
      if (c < N) {
        for (int h = 0; h < G; ++h) {
          const float u = X[(pp * G + h) * NP + c] - tau_s[pp * G + h];
          if (u > 0.f) pb += pow_pw(u, pw, kind);
        }
        pb /= (float)G;
      }
      const bool sel = pb > 0.f;
      const unsigned m = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int o = off + __popc(m & ((1u << lane) - 1u));
        idx[o] = cand_block(c, t, p.causal);
        logp[o] = logf(pb);
      }
      off += __popc(m);
    }
    if (lane == 0) p.cnt[row] = off;
  }

  // ---- optional per-head outputs
  if (p.tau || p.p_dense) {
    for (int r = warp; r < R; r += kThreads / 32) {
      const int pos = pos0 + r / G;
      if (pos >= p.S) continue;
      const int head = g * G + r % G;
      const int64_t hrow = ((int64_t)b * p.H + head) * p.S + pos;
      const float tau = N > 0 ? tau_s[r] : 0.f;
      if (p.tau && lane == 0) p.tau[hrow] = tau;
      if (p.p_dense) {
        float* pd = p.p_dense + hrow * p.t_cap;
        for (int cb = lane; cb < p.t_cap; cb += 32) {
          int ci = -1;
          if (p.causal) {
            ci = cb < t ? cb : -1;
          } else if (cb < T_ && cb != t) {
            ci = cb < t ? cb : cb - 1;
          }
          float v = 0.f;
          if (ci >= 0 && ci < N) {
            const float u = X[r * NP + ci] - tau;
            if (u > 0.f) v = pow_pw(u, pw, kind);
          }
          pd[cb] = v;
        }
      }
    }
  }
}

// Work list of a stage-2 tile of `tile_pos` consecutive positions: the union
// of the rows' selected blocks and the rows' own (diagonal) blocks,
// ascending; for each listed block, the bit mask of the tile positions that
// selected it; and the number of 64-token steps the tile takes (the causal
// diagonal's halves past the tile's last position are skipped).
// Second half of the tile work list (shared by the list and mask forms):
// pmask[c] holds the positions that selected block c; the list keeps those
// blocks and the tile's own blocks, ascending, and counts the tile's 64-token
// steps.  Warp 0 writes it.
__device__ __forceinline__ void emit_tile_list(const UnionParams& p, const uint4* pmask, int64_t bg, int tile,
                                               int pos0, int lane) {
  const int last = min(pos0 + p.tile_pos, p.S) - 1;
  const int own_lo = pos0 / p.block, own_hi = last / p.block;
  const int last_needed = p.causal ? last : p.S - 1;
  const int64_t tix = bg * p.n_tiles + tile;
  int32_t* out = p.ulist + tix * p.t_cap;
  uint4* mout = p.umask + tix * p.t_cap;
  int off = 0, steps = 0;
  for (int c0 = 0; c0 < p.t_cap; c0 += 32) {
    const int c = c0 + lane;
    bool keep = false;
    uint4 m = make_uint4(0u, 0u, 0u, 0u);
    if (c < p.t_cap) {
      m = pmask[c];
      keep = (m.x | m.y | m.z | m.w) != 0u || (c >= own_lo && c <= own_hi);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    int st = 0;
    if (keep) {
      const int k = off + __popc(bal & ((1u << lane) - 1u));
      out[k] = c;
      mout[k] = m;
      for (int h = 0; h < p.block / 64; ++h) st += (c * p.block + h * 64 <= last_needed) ? 1 : 0;
    }
    steps += warp_sum_i(st);
    off += __popc(bal);
  }
  if (lane == 0) {
    p.ucnt[tix] = off;
    p.usteps[tix] = steps;
  }
}

// Is block c a routing candidate of a row in block t?  (causal: an earlier
// block; otherwise any other block)
__device__ __forceinline__ bool candidate(const UnionParams& p, int c, int t, int n_blocks) {
  return c >= 0 && c != t && (p.causal ? c < t : c < n_blocks);
}

__global__ void __launch_bounds__(kThreads) union_kernel(UnionParams p) {
  extern __shared__ uint4 pmask[];  // [t_cap]: bit p set if tile position p selected the block
  const int b = blockIdx.z, g = blockIdx.y, tile = p.tile0 + blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int c = tid; c < p.t_cap; c += kThreads) pmask[c] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int pos0 = tile * p.tile_pos;
  const int n_blocks = (p.S + p.block - 1) / p.block;
  for (int pp = warp; pp < p.tile_pos; pp += kThreads / 32) {
    const int pos = pos0 + pp;
    if (pos >= p.S) break;
    const int t = pos / p.block;
    const int64_t row = bg * p.S + pos;
    const int n = min(max(p.cnt[row], 0), (int)p.t_cap);
    const int32_t* idx = p.idx + row * p.t_cap;
    for (int e = lane; e < n; e += 32) {
      const int c = idx[e];
      if (candidate(p, c, t, n_blocks)) {
        atomicOr(reinterpret_cast<uint32_t*>(&pmask[c]) + (pp >> 5), 1u << (pp & 31));
      } else {
        raise_status(p.status, 1 /* DASH_ERR_INVALID_ARGUMENT */, 200);
      }
    }
  }
  __syncthreads();
  if (warp == 0) emit_tile_list(p, pmask, bg, tile, pos0, lane);
}

// The same work list from bit-packed active-block masks (the pages' stage-2
// kernel iterates over such a mask): one warp per tile position walks its
// row's mask words, a lane per word, visiting the set bits with
// find-first-set; a set bit on a block that is not a candidate of the row (its
// own block, or a later one when causal) is skipped and reported.
__global__ void __launch_bounds__(kThreads) union_mask_kernel(UnionParams p) {
  extern __shared__ uint4 pmask[];
  const int b = blockIdx.z, g = blockIdx.y, tile = p.tile0 + blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int c = tid; c < p.t_cap; c += kThreads) pmask[c] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int pos0 = tile * p.tile_pos;
  const int n_blocks = (p.S + p.block - 1) / p.block;
  for (int pp = warp; pp < p.tile_pos; pp += kThreads / 32) {
    const int pos = pos0 + pp;
    if (pos >= p.S) break;
    const int t = pos / p.block;
    const uint32_t* words = p.mask + (bg * p.S + pos) * p.n_words;
    for (int w = lane; w < p.n_words; w += 32) {
      uint32_t word = __ldg(words + w);
      while (word) {
        const int c = 32 * w + __ffs(word) - 1;
        word &= word - 1u;
        if (c < p.t_cap && candidate(p, c, t, n_blocks)) {
          atomicOr(reinterpret_cast<uint32_t*>(&pmask[c]) + (pp >> 5), 1u << (pp & 31));
        } else {
          raise_status(p.status, 1 /* DASH_ERR_INVALID_ARGUMENT */, 201);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) emit_tile_list(p, pmask, bg, tile, pos0, lane);
}

// Work list of a pair of adjacent stage-2 tiles (see internal.h).
__global__ void __launch_bounds__(kThreads) pair_kernel(PairParams p) {
  extern __shared__ uint4 pm2[];  // [t_cap][2] masks, then [t_cap] presence bits
  uint32_t* pres = reinterpret_cast<uint32_t*>(pm2 + 2 * p.t_cap);
  const int b = blockIdx.z, g = blockIdx.y, pair = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int c = tid; c < p.t_cap; c += kThreads) {
    pm2[2 * c] = make_uint4(0u, 0u, 0u, 0u);
    pm2[2 * c + 1] = make_uint4(0u, 0u, 0u, 0u);
    pres[c] = 0u;
  }
  __syncthreads();
  const int64_t bg = (int64_t)b * p.Hkv + g;
  for (int t = 0; t < 2; ++t) {
    const int tile = 2 * pair + t;
    if (tile >= p.n_tiles) break;
    const int64_t tix = bg * p.n_tiles + tile;
    const int n = min(max(p.ucnt[tix], 0), (int)p.t_cap);
    for (int e = tid; e < n; e += kThreads) {
      const int c = p.ulist[tix * p.t_cap + e];
      if (c < 0 || c >= p.t_cap) continue;
      pm2[2 * c + t] = p.umask[tix * p.t_cap + e];
      atomicOr(&pres[c], 1u << t);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int pos0 = pair * 2 * p.tile_pos;
    const int last_needed = p.causal ? min(pos0 + 2 * p.tile_pos, p.S) - 1 : p.S - 1;
    const int64_t pix = bg * p.n_pairs + pair;
    int32_t* out = p.plist + pix * p.t_cap;
    uint4* mout = p.pmask + pix * p.t_cap * 2;
    int off = 0, steps = 0;
    for (int c0 = 0; c0 < p.t_cap; c0 += 32) {
      const int c = c0 + lane;
      const bool keep = c < p.t_cap && pres[c] != 0u;
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      int st = 0;
      if (keep) {
        const int k = off + __popc(bal & ((1u << lane) - 1u));
        out[k] = c;
        mout[2 * k] = pm2[2 * c];
        mout[2 * k + 1] = pm2[2 * c + 1];
        for (int h = 0; h < p.block / 64; ++h) st += (c * p.block + h * 64 <= last_needed) ? 1 : 0;
      }
      steps += warp_sum_i(st);
      off += __popc(bal);
    }
    if (lane == 0) {
      p.pcnt[pix] = off;
      p.psteps[pix] = steps;
    }
  }
}

template <typename T, int D>
cudaError_t launch_route_typed(const RouteParams& p, cudaStream_t stream) {
  const int T_ = (p.S + p.block - 1) / p.block;
  const int n_max = p.causal ? T_ - 1 : T_ - 1;
  const int np = (n_max + 3) & ~3;
  constexpr int DP = D + 4;
  const int smem_cap = 227 * 1024 - 1024;  // leave room for the static tau array
  int R = 64;
  int CW = 64;
  auto bytes = [&](int r, int cw) { return (size_t)(r * DP + cw * DP + r * np) * sizeof(float); };
  while (R > p.G && (R > 64 || bytes(R, CW) > (size_t)smem_cap)) {
    R /= 2;
    CW = 128;
  }
  if (R < p.G || R / p.G > p.block || bytes(R, CW) > (size_t)smem_cap) return cudaErrorInvalidValue;
  const size_t smem = bytes(R, CW);
  auto kern = route_prefill_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rpos = R / p.G;
  const int n_pos = p.S - p.pos_begin;
  if (n_pos <= 0) return cudaSuccess;
  dim3 grid((n_pos + rpos - 1) / rpos, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, stream>>>(p, R, CW);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_prefill(const RouteParams& p, cudaStream_t stream) {
  if (p.D == 128) {
    if (p.dtype == 0) return launch_route_typed<float, 128>(p, stream);
    if (p.dtype == 1) return launch_route_typed<__half, 128>(p, stream);
    return launch_route_typed<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 0) return launch_route_typed<float, 64>(p, stream);
  if (p.dtype == 1) return launch_route_typed<__half, 64>(p, stream);
  return launch_route_typed<__nv_bfloat16, 64>(p, stream);
}

cudaError_t launch_union(const UnionParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.t_cap * sizeof(uint4);
  auto kern = p.mask ? union_mask_kernel : union_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (p.n_tiles - p.tile0 <= 0) return cudaSuccess;
  dim3 grid(p.n_tiles - p.tile0, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_pairs(const PairParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.t_cap * (2 * sizeof(uint4) + sizeof(uint32_t));
  cudaError_t e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_pairs, p.Hkv, p.B);
  pair_kernel<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

// Bit-packed active-block masks (the pages' kernel walks a mask of the active
// chunks): one warp per row sets the bits of its listed blocks in a
// shared-memory copy of the row's words, then writes the words out.
namespace {
constexpr int kMaskWarps = 8;
constexpr int kMaskMaxWords = 128;  // t_cap <= 4096

__global__ void __launch_bounds__(kMaskWarps * 32)
    mask_kernel(const int32_t* idx, const int32_t* cnt, int64_t rows, int64_t t_cap, uint32_t* mask, int n_words) {
  __shared__ uint32_t words[kMaskWarps][kMaskMaxWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * kMaskWarps + warp; r < rows; r += (int64_t)gridDim.x * kMaskWarps) {
    for (int w = lane; w < n_words; w += 32) words[warp][w] = 0u;
    __syncwarp();
    const int n = min(max(cnt[r], 0), (int)t_cap);
    const int32_t* li = idx + r * t_cap;
    for (int i = lane; i < n; i += 32) {
      const int c = li[i];
      if (c >= 0 && c < n_words * 32) atomicOr(&words[warp][c >> 5], 1u << (c & 31));
    }
    __syncwarp();
    for (int w = lane; w < n_words; w += 32) mask[r * n_words + w] = words[warp][w];
    __syncwarp();
  }
}
}  // namespace

cudaError_t launch_lists_to_mask(const int32_t* idx, const int32_t* cnt, int64_t rows, int64_t t_cap,
                                 uint32_t* mask, int n_words, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (n_words > kMaskMaxWords) return cudaErrorInvalidValue;
  const int64_t want = (rows + kMaskWarps - 1) / kMaskWarps;
  const unsigned grid = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  mask_kernel<<<grid, kMaskWarps * 32, 0, stream>>>(idx, cnt, rows, t_cap, mask, n_words);
  return cudaGetLastError();
}

}  // namespace dash
