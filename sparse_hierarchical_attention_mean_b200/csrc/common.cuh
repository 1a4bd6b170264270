// Device helpers shared by the DashAttention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dash {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

// ---------------------------------------------------------------------------
// Element types: 16-byte vector loads converted to fp32.

template <typename T>
struct Elt;

template <>
struct Elt<float> {
  static constexpr int kPerVec = 4;
  __device__ static __forceinline__ void to_float(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ static __forceinline__ float load1(const float* p) { return *p; }
  __device__ static __forceinline__ void store1(float* p, float x) { *p = x; }
};

template <>
struct Elt<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static __forceinline__ void to_float(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

template <>
struct Elt<__half> {
  static constexpr int kPerVec = 8;
  __device__ static __forceinline__ void to_float(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 x = __half22float2(h);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  __device__ static __forceinline__ float load1(const __half* p) { return __half2float(*p); }
  __device__ static __forceinline__ void store1(__half* p, float x) { *p = __float2half_rn(x); }
};

// Pack two floats into a 32-bit pair of T (round to nearest even).
template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Warp reductions.

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ int warp_sum_i(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Reduce-scatter of NV per-lane partial sums across the warp.  On return,
// for NV >= 32 lane l holds the complete sums of indices l*(NV/32) + j in
// v[j] (j < NV/32); for NV < 32 it holds index l >> (5 - log2 NV) in v[0].
template <int NV>
__device__ __forceinline__ void warp_transpose_reduce(float* v, int lane) {
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n >= 2) {
      const int half = n / 2;
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < NV / 2; ++i) {
        if (i < half) {
          float send = upper ? v[i] : v[i + half];
          float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

// ---------------------------------------------------------------------------
// cp.async (16-byte, L2-only) with zero fill.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// alpha-entmax threshold of one row held in shared memory, solved by one
// warp.  x are the routing logits on the (alpha - 1) * z scale; the result
// tau satisfies sum_c [x_c - tau]_+^(1/(alpha-1)) = 1.
//
// Newton's method on F(tau) = sum [x - tau]_+^pw (convex and decreasing for
// pw >= 1) started at max(x) - 1, where F >= 1, approaches the root from
// below.  After every step the support S = {x > tau} is tested with the
// exact solution on S (sparsemax: linear; alpha = 1.5: quadratic); when that
// solution is self-consistent it is the answer.  Other alpha stop when the
// Newton step stalls.

__device__ __forceinline__ float pow_pw(float u, float pw, int kind) {
  // kind 0: pw == 1, kind 1: pw == 2, kind 2: general
  if (kind == 0) return u;
  if (kind == 1) return u * u;
  return exp2f(pw * log2f(u));
}

__device__ __forceinline__ int entmax_kind(float alpha) {
  return alpha == 2.0f ? 0 : (alpha == 1.5f ? 1 : 2);
}

// Newton passes from below with the exact check on the current support (see
// warp_entmax_tau).  SUBSET: each lane contributes the single value v;
// otherwise the row is x[c] for c < n, strided over the lanes.  tau must be a
// lower bound of the root (F(tau) >= 1).
template <bool SUBSET>
__device__ inline float entmax_newton(const float* x, float v, int n, float tau, float pw, int kind, int lane) {
  for (int it = 0; it < 100; ++it) {
    float f = 0.f, fd = 0.f, a = 0.f, umin = 3.0e38f;
    int k = 0;
    for (int c = SUBSET ? 0 : lane; c < (SUBSET ? 1 : n); c += 32) {
      const float u = (SUBSET ? v : x[c]) - tau;
      if (u > 0.f) {
        ++k;
        a += u;
        umin = fminf(umin, u);
        if (kind == 0) {
          f += u;
        } else if (kind == 1) {
          f += u * u;
        } else {
          const float up = exp2f((pw - 1.0f) * log2f(u));
          fd += up;
          f += up * u;
        }
      }
    }
    f = warp_sum(f);
    a = warp_sum(a);
    k = warp_sum_i(k);
    umin = warp_min(umin);
    if (kind == 0) {
      // exact on the support: tau' = tau + (F - 1) / k
      const float delta = (f - 1.0f) / (float)k;
      if (delta < umin) return tau + fmaxf(delta, 0.0f);
      tau += delta;  // Newton step == exact step; support shrinks
    } else if (kind == 1) {
      // exact on the support: k d^2 - 2 A d + (F - 1) = 0, smaller root
      const float disc = a * a - (float)k * (f - 1.0f);
      if (disc >= 0.f) {
        const float delta = (f - 1.0f) / (a + sqrtf(disc));  // = (A - sqrt(disc)) / k
        if (delta < umin) return tau + fmaxf(delta, 0.0f);
      }
      tau += (f - 1.0f) / (2.0f * a);  // Newton
    } else {
      fd = warp_sum(fd);
      const float step = (f - 1.0f) / (pw * fd);
      tau += step;
      if (fabsf(step) <= 1e-7f * fmaxf(1.0f, fabsf(tau))) return tau;
    }
  }
  return tau;
}

// alpha-entmax threshold of one row x[0..n) by one warp.  F(tau) =
// sum_c [x_c - tau]_+^(1/(alpha-1)) is convex and decreasing, F(max - 1) >= 1,
// so Newton from below approaches the root monotonically; after every step
// the exact solution on the current support (linear for sparsemax, quadratic
// for alpha = 1.5) is accepted when it is self-consistent.  The start is the
// threshold of the 32 lane maxima, solved first in registers: they are a
// subset of the row and F over a subset is below F over the row, so that
// threshold is a lower bound too, and usually one pass over the row from
// there finds the exact support.
__device__ inline float warp_entmax_tau(const float* x, int n, float alpha, int lane) {
  const float pw = 1.0f / (alpha - 1.0f);
  const int kind = entmax_kind(alpha);
  float lm = kNegInf;
  for (int c = lane; c < n; c += 32) lm = fmaxf(lm, x[c]);
  const float mx = warp_max(lm);
  float tau = mx - 1.0f;
  if (mx == kNegInf) return tau;
  tau = entmax_newton<true>(nullptr, lm, 1, tau, pw, kind, lane);
  return entmax_newton<false>(x, 0.f, n, tau, pw, kind, lane);
}

// Status word kept in the first bytes of every workspace.
struct DeviceStatus {
  int32_t code;    // 0 ok, else a dash_status_t
  int32_t detail;  // where it was raised
};

__device__ __forceinline__ void raise_status(DeviceStatus* st, int code, int detail) {
  if (st) {
    if (atomicCAS(&st->code, 0, code) == 0) st->detail = detail;
  }
}

}  // namespace dash
