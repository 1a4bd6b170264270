// Stage 0: block summaries s_c = mean_{j in c} k_j @ W_s.
//
// "Stage 0: local chunk summary" of the DashAttention technical summary: the
// context is cut into contiguous chunks and each chunk is summarised once
// (and cached once complete).  The learned summary query starts at zero,
// which is uniform mean pooling; here the summary is the block mean followed
// by the fixed projection W_s (row vector times matrix).
//
// HBM-bound: every key is read once with 16-byte vector loads; the mean and
// the projection are fp32.  One CTA pools `bpc` consecutive blocks of one
// (batch, KV head) and projects them together so each W_s column is read
// once per CTA.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxBpc = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) pool_kernel(PoolParams p, int bpc) {
  constexpr int EPV = Elt<T>::kPerVec;
  constexpr int VPR = D / EPV;        // 16-byte vectors per key row
  constexpr int RP = kThreads / VPR;  // key rows per pass
  constexpr int NG = kThreads / D;    // thread groups in the projection
  __shared__ float red[RP][D];
  __shared__ float means[kMaxBpc][D];

  const int b = blockIdx.z, g = blockIdx.y;
  int n_tok = p.S;
  if (p.seqlens) n_tok = min(max(p.seqlens[b], 0), p.S);
  const int64_t nblk = (n_tok + p.block - 1) / p.block;
  const int64_t c_begin = p.first_block + (int64_t)blockIdx.x * bpc;
  if (c_begin >= nblk) return;
  const int nb = (int)(nblk - c_begin < bpc ? nblk - c_begin : bpc);
  const int tid = threadIdx.x;
  const int vrow = tid / VPR, vcol = tid % VPR;
  const T* kbase = static_cast<const T*>(p.k.data) + (int64_t)b * p.k.sb + (int64_t)g * p.k.sh + vcol * EPV;

  for (int i = 0; i < nb; ++i) {
    const int64_t lo = (c_begin + i) * p.block;
    const int64_t hi = lo + p.block < n_tok ? lo + p.block : (int64_t)n_tok;
    float acc[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
#pragma unroll 8
    for (int64_t j = lo + vrow; j < hi; j += RP) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(kbase + j * p.k.ss));
      float f[EPV];
      Elt<T>::to_float(v, f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[e] += f[e];
    }
#pragma unroll
    for (int e = 0; e < EPV; ++e) red[vrow][vcol * EPV + e] = acc[e];
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < RP; ++r) s += red[r][tid];
      means[i][tid] = s / (float)(hi - lo);
    }
    __syncthreads();
  }

  // s[i][col] = sum_k mean[i][k] * W_s[k][col]
  const int col = tid % D, grp = tid / D;
  constexpr int PER = kMaxBpc / NG;
  float acc[PER];
#pragma unroll
  for (int m = 0; m < PER; ++m) acc[m] = 0.f;
  for (int k = 0; k < D; ++k) {
    const float w = __ldg(p.w_s + k * D + col);
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int i = grp + NG * m;
      if (i < nb) acc[m] += means[i][k] * w;
    }
  }
  float* out = p.summaries + ((int64_t)b * p.Hkv + g) * p.t_cap * D;
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    const int i = grp + NG * m;
    if (i < nb) out[(c_begin + i) * D + col] = acc[m];
  }
}

template <typename T, int D>
cudaError_t launch_typed(const PoolParams& p, cudaStream_t stream) {
  const int64_t max_blk = (p.S + p.block - 1) / p.block;
  const int64_t span = max_blk - p.first_block;
  if (span <= 0) return cudaSuccess;
  const int64_t total = span * p.B * p.Hkv;
  int bpc = 4;
  while (bpc < kMaxBpc && total / (bpc * 2) >= 148 * 16) bpc *= 2;
  dim3 grid((unsigned)((span + bpc - 1) / bpc), p.Hkv, p.B);
  pool_kernel<T, D><<<grid, kThreads, 0, stream>>>(p, bpc);
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
