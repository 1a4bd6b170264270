// Stage 0: block summaries s_c = mean_{j in c} k_j @ W_s.
//
// "Stage 0: local chunk summary" of the DashAttention technical summary: the
// context is cut into contiguous chunks and each chunk is summarised once
// (and cached once complete).  The learned summary query starts at zero,
// which is uniform mean pooling; here the summary is the block mean followed
// by the fixed projection W_s (row vector times matrix).
//
// With a learned summary query q_bar (one per KV head) the block's keys are
// weighted by softmax_j(q_bar . k_j / sqrt(d)) instead of uniformly; q_bar = 0
// is the mean (the pages' zero initialisation).
//
// HBM-bound: every key is read once with 16-byte vector loads; the mean and
// the projection are fp32.  One CTA pools up to 32 consecutive blocks of one
// (batch, KV head) and projects them together so each W_s row is read once
// per CTA.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsP = kThreads / 32;
constexpr int kMaxBpc = 32;

// One CTA: up to kMaxBpc consecutive blocks of one (batch, KV head).
//   Pooling: each warp takes whole blocks (w, w + 8, ...); a lane owns one
//   16-byte column vector of a row group and sums its rows in registers with
//   sixteen loads in flight (mean pooling; eight with the learned query),
//   then the lanes holding the same columns combine by shuffles.  No barrier
//   per block.
//   Projection: means[nb][D] x W_s[D][D] with a 4 x 4 (blocks x columns)
//   register tile per thread; W_s rows are read as float4 through L1.
template <typename T, int D, bool SDPA>
__global__ void __launch_bounds__(kThreads) pool_kernel(PoolParams p, int bpc) {
  constexpr int EPV = Elt<T>::kPerVec;     // elements per 16-byte vector
  constexpr int VPR = D / EPV;             // vectors per key row (8, 16 or 32)
  constexpr int RPL = 32 / VPR;            // rows per warp-wide load
  constexpr int CG = D / 4;                // 4-column groups of the projection
  constexpr int BG = kThreads / CG;        // block groups
  constexpr int BPT = kMaxBpc / BG;        // blocks per thread in the projection
  __shared__ __align__(16) float means[kMaxBpc][D];

  // consecutive CTAs take the same blocks of consecutive KV heads: the heads'
  // rows of a token are adjacent in memory, so the CTAs in flight together
  // read whole rows of the cache and each DRAM page is opened once
  const int b = blockIdx.z;
  const int g = (int)(blockIdx.x % (unsigned)p.Hkv);
  const int chunk = (int)(blockIdx.x / (unsigned)p.Hkv);
  int n_tok = p.S;
  if (p.seqlens) n_tok = min(max(p.seqlens[b], 0), p.S);
  const int64_t nblk = (n_tok + p.block - 1) / p.block;
  const int64_t c_begin = p.first_block + (int64_t)chunk * bpc;
  if (c_begin >= nblk) return;
  const int nb = (int)(nblk - c_begin < bpc ? nblk - c_begin : bpc);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int vcol = lane % VPR, vrow = lane / VPR;
  const T* kbase = static_cast<const T*>(p.k.data) + (int64_t)g * p.k.sh + vcol * EPV;
  // rows of block c: row j (absolute token) at block_base(c) + (j - c * block) * ss
  auto block_base = [&](int64_t c) -> const T* {
    if (p.block_table) return kbase + (int64_t)p.block_table[(int64_t)b * p.max_blocks + c] * p.k.sb;
    return kbase + (int64_t)b * p.k.sb + c * p.block * p.k.ss;
  };

  if constexpr (!SDPA) {
    for (int i = warp; i < nb; i += kWarpsP) {
      const int64_t lo = (c_begin + i) * p.block;
      const int64_t hi = lo + p.block < n_tok ? lo + p.block : (int64_t)n_tok;
      const T* kb = block_base(c_begin + i);
      float acc[EPV];
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
      for (int64_t j0 = lo; j0 < hi; j0 += 16 * RPL) {
        uint4 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int64_t j = j0 + u * RPL + vrow;
          v[u] = j < hi ? __ldg(reinterpret_cast<const uint4*>(kb + (j - lo) * p.k.ss)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float f[EPV];
          Elt<T>::to_float(v[u], f);
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[e] += f[e];
        }
      }
#pragma unroll
      for (int off = VPR; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
      if (vrow == 0) {
        const float inv = 1.0f / (float)(hi - lo);
#pragma unroll
        for (int e = 0; e < EPV; ++e) means[i][vcol * EPV + e] = acc[e] * inv;
      }
    }
  } else {
    // learned summary query: weights softmax_j(q_bar . k_j / sqrt(D)) over the
    // block.  Each lane keeps an online softmax (reference max, denominator,
    // weighted key sum) over its rows; the row score is the sum of the
    // partial dot products of the VPR lanes holding the row; the lanes of
    // the block merge at the end.  Scores are in the log2 domain.
    float qv[EPV];
    {
      const float sc = rsqrtf((float)D) * kLog2e;
      const float* qb = p.qbar + (int64_t)g * D + vcol * EPV;
#pragma unroll
      for (int e = 0; e < EPV; ++e) qv[e] = __ldg(qb + e) * sc;
    }
    for (int i = warp; i < nb; i += kWarpsP) {
      const int64_t lo = (c_begin + i) * p.block;
      const int64_t hi = lo + p.block < n_tok ? lo + p.block : (int64_t)n_tok;
      const T* kb = block_base(c_begin + i);
      float acc[EPV], m = kNegInf, den = 0.f;
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
      for (int64_t j0 = lo; j0 < hi; j0 += 8 * RPL) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t j = j0 + u * RPL + vrow;
          v[u] = j < hi ? __ldg(reinterpret_cast<const uint4*>(kb + (j - lo) * p.k.ss)) : make_uint4(0u, 0u, 0u, 0u);
        }
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float f[EPV];
          Elt<T>::to_float(v[u], f);
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < EPV; ++e) d = fmaf(qv[e], f[e], d);
          a[u] = d;
        }
#pragma unroll
        for (int off = 1; off < VPR; off <<= 1)
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] += __shfl_xor_sync(0xffffffffu, a[u], off);
        float mr = m;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u * RPL + vrow >= hi) a[u] = kNegInf;
          mr = fmaxf(mr, a[u]);
        }
        const float ms = mr == kNegInf ? 0.f : mr;
        const float corr = exp2f(m - ms);
        den *= corr;
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[e] *= corr;
        m = mr;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = exp2f(a[u] - ms);
          float f[EPV];
          Elt<T>::to_float(v[u], f);
          den += w;
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[e] = fmaf(w, f[e], acc[e]);
        }
      }
      // merge the lanes that hold the same columns (different rows)
#pragma unroll
      for (int off = VPR; off < 32; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
        const float dn = __shfl_xor_sync(0xffffffffu, den, off);
        const float mm = fmaxf(m, mo);
        const float ms = mm == kNegInf ? 0.f : mm;
        const float c0 = exp2f(m - ms), c1 = exp2f(mo - ms);
        den = den * c0 + dn * c1;
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[e] = acc[e] * c0 + __shfl_xor_sync(0xffffffffu, acc[e], off) * c1;
        m = mm;
      }
      if (vrow == 0) {
        const float inv = 1.0f / den;
#pragma unroll
        for (int e = 0; e < EPV; ++e) means[i][vcol * EPV + e] = acc[e] * inv;
      }
    }
  }
  __syncthreads();

  // s[i][col] = sum_k mean[i][k] * W_s[k][col]
  const int cg = tid % CG, bgp = tid / CG;
  float acc[BPT][4];
#pragma unroll
  for (int m = 0; m < BPT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
  const float4* w4 = reinterpret_cast<const float4*>(p.w_s) + cg;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    const float4 w = __ldg(w4 + k * (D / 4));
#pragma unroll
    for (int m = 0; m < BPT; ++m) {
      const float mk = means[bgp * BPT + m][k];
      acc[m][0] = fmaf(mk, w.x, acc[m][0]);
      acc[m][1] = fmaf(mk, w.y, acc[m][1]);
      acc[m][2] = fmaf(mk, w.z, acc[m][2]);
      acc[m][3] = fmaf(mk, w.w, acc[m][3]);
    }
  }
  float* out = p.summaries + ((int64_t)b * p.Hkv + g) * p.t_cap * D;
#pragma unroll
  for (int m = 0; m < BPT; ++m) {
    const int i = bgp * BPT + m;
    if (i < nb)
      *reinterpret_cast<float4*>(out + (c_begin + i) * D + cg * 4) =
          make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
  }
}

template <typename T, int D>
cudaError_t launch_typed(const PoolParams& p, cudaStream_t stream) {
  const int64_t max_blk = (p.S + p.block - 1) / p.block;
  const int64_t span = max_blk - p.first_block;
  if (span <= 0) return cudaSuccess;
  const int64_t total = span * p.B * p.Hkv;
  // as many blocks per CTA as keep about four CTAs per SM busy
  int bpc = kMaxBpc;
  while (bpc > kWarpsP && total / bpc < 148 * 4) bpc /= 2;
  dim3 grid((unsigned)((span + bpc - 1) / bpc * p.Hkv), 1, p.B);
  if (p.qbar)
    pool_kernel<T, D, true><<<grid, kThreads, 0, stream>>>(p, bpc);
  else
    pool_kernel<T, D, false><<<grid, kThreads, 0, stream>>>(p, bpc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const PoolParams& p, cudaStream_t stream) {
  if (p.D == 128) {
    if (p.dtype == 0) return launch_typed<float, 128>(p, stream);
    if (p.dtype == 1) return launch_typed<__half, 128>(p, stream);
    return launch_typed<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 0) return launch_typed<float, 64>(p, stream);
  if (p.dtype == 1) return launch_typed<__half, 64>(p, stream);
  return launch_typed<__nv_bfloat16, 64>(p, stream);
}

}  // namespace dash
