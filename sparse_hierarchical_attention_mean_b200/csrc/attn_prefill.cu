// Stage 2 for prefill with fp32 inputs: prior-induced sparse softmax on the
// CUDA cores.
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: softmax is the maximiser of <p, l> - KL(p || u); replacing the
// uniform reference u by a prior g built from the routing weights gives
// softmax(l + log g), and g = 0 on blocks with zero routing mass masks them.
// The near-diagonal block has no summary and is always included (prior
// log(1/N), causal mask).  One warp per (position, head) row walks the row's
// own ascending block list, then the diagonal block, in fp32.  The f16/bf16
// path is the tensor-core kernel in attn_prefill_tc.cu.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

// ---------------------------------------------------------------- fp32 CUDA-core path
template <int D>
__global__ void __launch_bounds__(256) sparse_simt_kernel(SparseParams p) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row_id = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int b = blockIdx.y;
  if (row_id >= (int64_t)p.S * p.H) return;
  const int pos = (int)(row_id / p.H), head = (int)(row_id % p.H);
  const int g = head / p.G;
  const int t = pos / p.block;
  const int T_ = (p.S + p.block - 1) / p.block;
  const int N = p.causal ? t : T_ - 1;
  const int64_t lrow = ((int64_t)b * p.Hkv + g) * p.S + pos;
  const int n = min(max(p.cnt[lrow], 0), (int)p.t_cap);
  const int32_t* idx = p.idx + lrow * p.t_cap;
  const float* logp = p.logp + lrow * p.t_cap;
  const float* q = static_cast<const float*>(p.q.data) + b * p.q.sb + pos * p.q.ss + head * p.q.sh;
  const float* kg = static_cast<const float*>(p.k.data) + b * p.k.sb + g * p.k.sh;
  const float* vg = static_cast<const float*>(p.v.data) + b * p.v.sb + g * p.v.sh;
  float qr[DL], o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) {
    qr[e] = q[lane * DL + e] * rsqrtf((float)D);
    o[e] = 0.f;
  }
  float m = kNegInf, l = 0.f;
  const float beta = N > 0 ? p.sigma * logf(1.0f / (float)N) : 0.0f;
  for (int it = 0; it <= n; ++it) {
    const bool diag = it == n;
    const int c = diag ? t : idx[it];
    if (!diag && (c < 0 || c == t || (p.causal ? c >= t : c >= T_))) {
      raise_status(p.status, 1 /* DASH_ERR_INVALID_ARGUMENT */, 201);
      continue;
    }
    const float bias = diag ? beta : p.sigma * logp[it];
    const int lo = c * p.block;
    int hi = min(lo + p.block, p.S);
    if (diag && p.causal) hi = pos + 1;
    for (int j = lo; j < hi; ++j) {
      const float* kj = kg + (int64_t)j * p.k.ss + lane * DL;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) s = fmaf(qr[e], kj[e], s);
      s = warp_sum(s) + bias;
      const float mn = fmaxf(m, s);
      const float sc = expf(m - mn);
      const float pj = expf(s - mn);
      l = l * sc + pj;
      const float* vj = vg + (int64_t)j * p.v.ss + lane * DL;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[e] = o[e] * sc + pj * vj[e];
      m = mn;
    }
  }
  float* out = static_cast<float*>(const_cast<void*>(p.out.data)) + b * p.out.sb + pos * p.out.ss + head * p.out.sh;
#pragma unroll
  for (int e = 0; e < DL; ++e) out[lane * DL + e] = o[e] / l;
}

}  // namespace

int sparse_tile_positions(int G, int /*block*/) { return 128 / G; }

cudaError_t launch_sparse_prefill(const SparseParams& p, cudaStream_t stream) {
  if (p.dtype != 0) return launch_sparse_prefill_tc(p, stream);
  dim3 grid((unsigned)(((int64_t)p.S * p.H + 7) / 8), p.B);
  if (p.D == 128)
    sparse_simt_kernel<128><<<grid, 256, 0, stream>>>(p);
  else
    sparse_simt_kernel<64><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dash
