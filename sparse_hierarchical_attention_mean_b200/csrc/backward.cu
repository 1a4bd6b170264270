// Backward pass of the prefill forward: gradients of sum(dout * out) with
// respect to q, k, v and W_s.
//
// "Stage 1: entmax chunk routing" of the DashAttention technical summary
// makes the router differentiable: the prior log p_bar of "Stage 2:
// prior-induced sparse softmax" passes the attention gradient back through
// the GQA mean and the alpha-entmax Jacobian (Peters, Niculae & Martins 2019,
// section 3: dp/dz = diag(u) - u u^T / sum(u), u = p^(2 - alpha) on the
// support) to the block scores, and from there to the queries and to the
// block summaries of "Stage 0: local chunk summary".
//
// The call (dash_attn_bwd) first recomputes the forward's summaries, lists and
// per-head thresholds, runs the forward's stage-2 kernel for each row's
// log-sum-exp, and builds bit masks of the rows' selections and of the
// stage-2 tiles' work lists.  Then, in order:
//   row (bwd_row_tc.cu)  one CTA per stage-2 tile on the tensor cores: D =
//              dout . out, dS = P (dP - D), dq = dS K / sqrt(d) and each row's
//              d log p_bar of every selected block, per head (into dz);
//   bwd_route  one CTA per (row, KV head), here: the entmax vector-Jacobian
//              product per head from the recomputed scores and the
//              forward's thresholds (dz becomes dL/dz), and dq += gamma dz S;
//   key (bwd_key_tc.cu)  one CTA per 128 keys on the tensor cores: dk, dv,
//              the summary gradient ds = gamma sum dz q, the stage-0 term
//              ds W_s^T / |c| in dk and the block means;
//   bwd_ws     here: dW_s = sum over blocks of kbar^T ds.
// No atomics: every gradient element has one writer, so results are
// reproducible run to run.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

// ------------------------------------------------------------------ bwd_route
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) bwd_route_kernel(BwdParams p) {
  extern __shared__ __align__(16) float rsm[];
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.S;
  const int64_t tc = p.t_cap;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int64_t row = bg * S + r;
  const int n = p.cnt[row];
  if (n <= 0) return;
  float* qs = rsm;          // [G][D]
  float* gv = qs + G * D;   // [t_cap] dL/dp of each entry (same for every head)
  float* u = gv + tc;        // [G][t_cap] u, then dL/dz
  float* red = u + G * tc;   // [4][2 G]
  for (int i = tid; i < G * D; i += 128) {
    const int hh = i / D, c = i - hh * D;
    qs[i] = Elt<T>::load1(static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)r * p.q.ss +
                          (int64_t)(g * G + hh) * p.q.sh + c);
  }
  const int32_t* list = p.idx + row * tc;
  const float* lp = p.logp + row * tc;
  float* dz = p.dz + row * tc * G;
  // through log and the mean over the G heads: dp_h = d log p_bar / (G p_bar)
  for (int e = tid; e < n; e += 128) {
    float s = 0.f;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) s += dz[e * G + hh];
    gv[e] = s / ((float)G * expf(lp[e]));
  }
  __syncthreads();
  const float gam = rsqrtf((float)D);
  const float a1 = p.alpha - 1.0f;
  const float upw = (2.0f - p.alpha) / a1;
  const int kind = entmax_kind(p.alpha);
  float su[G], sug[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) su[hh] = sug[hh] = 0.f;
  for (int e = tid; e < n; e += 128) {
    const float4* srow = reinterpret_cast<const float4*>(p.summaries + (bg * tc + list[e]) * D);
    float z[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) z[hh] = 0.f;
    for (int k4 = 0; k4 < D / 4; ++k4) {
      const float4 s4 = __ldg(srow + k4);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float* qh = qs + hh * D + 4 * k4;
        z[hh] = fmaf(qh[0], s4.x, fmaf(qh[1], s4.y, fmaf(qh[2], s4.z, fmaf(qh[3], s4.w, z[hh]))));
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      // x - tau on the (alpha - 1) z scale; u = p^(2 - alpha) = (x - tau)^((2 - alpha)/(alpha - 1))
      const float xm = a1 * gam * z[hh] - p.tau[((int64_t)b * p.H + g * G + hh) * S + r];
      const float uu = xm > 0.f ? (kind == 0 ? 1.0f : kind == 1 ? xm : powf(xm, upw)) : 0.f;
      u[hh * tc + e] = uu;
      su[hh] += uu;
      sug[hh] += uu * gv[e];
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    su[hh] = warp_sum(su[hh]);
    sug[hh] = warp_sum(sug[hh]);
    if (lane == 0) {
      red[warp * 2 * G + hh] = su[hh];
      red[warp * 2 * G + G + hh] = sug[hh];
    }
  }
  __syncthreads();
  float ghat[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float s1 = red[hh] + red[2 * G + hh] + red[4 * G + hh] + red[6 * G + hh];
    const float s2 = red[G + hh] + red[3 * G + hh] + red[5 * G + hh] + red[7 * G + hh];
    ghat[hh] = s1 > 0.f ? s2 / s1 : 0.f;
  }
  for (int e = tid; e < n; e += 128) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float v = u[hh * tc + e] * (gv[e] - ghat[hh]);
      u[hh * tc + e] = v;
      dz[e * G + hh] = v;
    }
  }
  __syncthreads();
  if (tid < D) {
    float acc[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) acc[hh] = 0.f;
    for (int e = 0; e < n; ++e) {
      const float sv = __ldg(p.summaries + (bg * tc + list[e]) * D + tid);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) acc[hh] = fmaf(u[hh * tc + e], sv, acc[hh]);
    }
    float* dqg = static_cast<float*>(const_cast<void*>(p.dq.data)) + (int64_t)b * p.dq.sb + (int64_t)r * p.dq.ss + tid;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) dqg[(int64_t)(g * G + hh) * p.dq.sh] += gam * acc[hh];
  }
}

// ------------------------------------------------------------------ bwd_ws
// dW_s[a][col] = sum over blocks i of kbar[i][a] ds[i][col]; one CTA per row a.
__global__ void bwd_ws_kernel(const float* __restrict__ kbar, const float* __restrict__ ds, int64_t n, int D,
                              float* __restrict__ dw) {
  const int a = blockIdx.x, col = threadIdx.x;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int64_t i = 0;
  for (; i + 4 <= n; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = fmaf(kbar[(i + u) * D + a], ds[(i + u) * D + col], acc[u]);
  for (; i < n; ++i) acc[0] = fmaf(kbar[i * D + a], ds[i * D + col], acc[0]);
  dw[(int64_t)a * D + col] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <typename T, int D>
cudaError_t launch_typed(const BwdParams& p, cudaStream_t stream) {
  // dq of stage 2, d log p_bar per head and D on the tensor cores
  cudaError_t e = launch_bwd_row_tc(p, stream);
  if (e != cudaSuccess) return e;

  const size_t route_smem = (size_t)(p.G * D + p.t_cap + (int64_t)p.G * p.t_cap + 8 * p.G) * 4;
  auto launch_route = [&](auto kernel) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)route_smem);
    if (err != cudaSuccess) return err;
    kernel<<<dim3(p.S, p.Hkv, p.B), 128, route_smem, stream>>>(p);
    return cudaGetLastError();
  };
  switch (p.G) {
    case 1: e = launch_route(bwd_route_kernel<T, D, 1>); break;
    case 2: e = launch_route(bwd_route_kernel<T, D, 2>); break;
    case 4: e = launch_route(bwd_route_kernel<T, D, 4>); break;
    default: e = launch_route(bwd_route_kernel<T, D, 8>); break;
  }
  if (e != cudaSuccess) return e;

  // dk, dv, the summary gradient and the block means on the tensor cores
  if ((e = launch_bwd_key_tc(p, stream)) != cudaSuccess) return e;

  bwd_ws_kernel<<<D, D, 0, stream>>>(p.kbar, p.ds, (int64_t)p.B * p.Hkv * p.t_cap, D, p.dw_s);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dtype(const BwdParams& p, cudaStream_t stream) {
  return p.D == 128 ? launch_typed<T, 128>(p, stream) : launch_typed<T, 64>(p, stream);
}

}  // namespace

cudaError_t launch_bwd(const BwdParams& p, cudaStream_t stream) {
  if (p.dtype == 1) return launch_dtype<__half>(p, stream);
  return launch_dtype<__nv_bfloat16>(p, stream);
}

}  // namespace dash
