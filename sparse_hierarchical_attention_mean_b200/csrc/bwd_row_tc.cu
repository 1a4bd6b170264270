// Row-centric backward on the 5th-generation tensor cores: the stage-2 part
// of dq, each row's gradient of its prior log p_bar (d log p_bar, per head)
// and D = dout . out.
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: o = sum_j P_j v_j with P = softmax(q k^T / sqrt(d) + bias), the
// bias sigma * log p_bar_c on the tokens of a selected block c and
// sigma * log(1/N) on the diagonal block.  With D = dout . o and
// dS_j = P_j (dout . v_j - D):  dq = sum_j dS_j k_j / sqrt(d), and, the bias
// of block c being sigma * log p_bar_c, d log p_bar_c = sigma sum_{j in c} dS_j
// ("Stage 1: entmax chunk routing" carries it on through the GQA mean and the
// alpha-entmax Jacobian).
//
// One CTA per stage-2 tile (128 rows: 128 / G positions x G heads of one KV
// group), walking the tile's work list (its blocks in 64-token steps, as the
// forward does) with each row's log-sum-exp from the forward's stage-2 kernel:
//   S  = Q K^T    (TS MMA, A = Q from TMEM)       } double-buffered in TMEM,
//   dP = dout V^T (TS MMA, A = dout from TMEM)    } the next step's run while
//   P = 2^(S scale + bias - lse), dS = P (dP - D)    this step's softmax does
//   dQ += dS K    (TS MMA, A = dS written packed over S, K MN-major)
// Warps 0-3 own the rows (TMEM lanes): they store Q and dout into TMEM, form
// D, P and dS, sum dS over each selected block and write dq at the end; warp
// 4 streams K and V (TMA, 4-D maps, 128-byte swizzle, no multicast); warp 5
// issues the MMAs.  Every mbarrier wait is bounded; on expiry the kernel
// records DASH_ERR_DEVICE_TIMEOUT and winds down.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace dash {
namespace {

constexpr int kRowsR = 128;
constexpr int kStepR = 64;  // keys per step
constexpr int kProdWarpR = 4;
constexpr int kMmaWarpR = 5;
constexpr int kThreadsR = 192;
constexpr int kMaxStagesR = 8;

template <int D>
struct RowLayout {
  static constexpr int KC = D / 64;
  static constexpr int kKVChunk = kStepR * 128;  // 8 KB
  static constexpr int kKVBytes = KC * kKVChunk;
  static constexpr int kStages = D == 128 ? 6 : 8;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  static constexpr int kBytes = kOffBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
  // TMEM columns: Q and dout (16-bit pairs), two S / dP buffers, dQ
  static constexpr uint32_t kColQ = 0, kColO = D / 2, kColSD = D;  // buffer b: S at kColSD + 128 b, dP + 64
  static constexpr uint32_t kColDQ = D + 256;
};

struct StepR {
  int c, tok0, first, last;  // block, first token, first / last step of the block
  uint4 mask;                // tile positions that selected the block
};

struct RBarsB {
  uint64_t qo_full;  // Q and dout stored into TMEM (128 arrivals)
  uint64_t kv_full[kMaxStagesR];
  uint64_t kv_empty[kMaxStagesR];
  uint64_t s_full[2];
  uint64_t p_full[2];  // 128 arrivals
  uint64_t dq_final;
  uint32_t tmem_base;
  int abort;
  StepR desc[kMaxStagesR];
};

__device__ __forceinline__ void failr(RBarsB* bars, DeviceStatus* st, int where) {
  raise_status(st, 5 /* DASH_ERR_DEVICE_TIMEOUT */, where);
  atomicExch(&bars->abort, 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreadsR, 1)
    bwd_row_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdParams p) {
  using L = RowLayout<D>;
  constexpr int kStages = L::kStages;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = tc::idesc_f16(kRowsR, kStepR, kBF16, false, false);
  constexpr uint32_t kIdescQ = tc::idesc_f16(kRowsR, D, kBF16, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RBarsB* bars = reinterpret_cast<RBarsB*>(smem + L::kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = p.G;
  const int P = kRowsR / G;
  const int pos0 = tile * P;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int64_t tix = bg * p.n_tiles + tile;
  const int32_t* list = p.ulist + tix * p.t_cap;
  const uint4* lmask = p.tmask + tix * p.t_cap;
  const int n_list = min(max(p.ucnt[tix], 0), (int)p.t_cap);
  const int n_steps = p.usteps[tix];

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->qo_full, kRowsR);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], kRowsR);
    }
    tc::mbar_init(&bars->dq_final, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarpR) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == kProdWarpR && lane == 0) {
    tc::prefetch_tensormap(&tm_k);
    tc::prefetch_tensormap(&tm_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kProdWarpR) {
    // ------------------------------------------------------------ producer
    const int spb = p.block / kStepR;
    const int last_needed = p.causal ? min(pos0 + P, p.S) - 1 : p.S - 1;
    int i = 0;
    bool ok = true;
    for (int u0 = 0; ok && u0 < n_list; u0 += 32) {
      const bool have = u0 + lane < n_list;
      const int my_c = have ? __ldg(list + u0 + lane) : 0;
      const uint4 my_m = have ? __ldg(lmask + u0 + lane) : make_uint4(0u, 0u, 0u, 0u);
      const int nj = min(32, n_list - u0);
      for (int j = 0; ok && j < nj; ++j) {
        const int c = __shfl_sync(0xffffffffu, my_c, j);
        uint4 m;
        m.x = __shfl_sync(0xffffffffu, my_m.x, j);
        m.y = __shfl_sync(0xffffffffu, my_m.y, j);
        m.z = __shfl_sync(0xffffffffu, my_m.z, j);
        m.w = __shfl_sync(0xffffffffu, my_m.w, j);
        int n_h = 0;  // steps of this block the tile takes
        for (int h = 0; h < spb; ++h) n_h += (c * p.block + h * kStepR <= last_needed) ? 1 : 0;
        for (int h = 0; h < n_h; ++h) {
          const int tok0 = c * p.block + h * kStepR;
          if (lane == 0) {
            const int st = i % kStages;
            if (i >= kStages && !tc::mbar_wait(&bars->kv_empty[st], ((i / kStages) - 1) & 1)) {
              failr(bars, p.status, 50);
              ok = false;
            } else {
              StepR& d = bars->desc[st];
              d.c = c;
              d.tok0 = tok0;
              d.first = h == 0;
              d.last = h == n_h - 1;
              d.mask = m;
              tc::mbar_arrive_expect_tx(&bars->kv_full[st], 2 * L::kKVBytes);
              for (int kc = 0; kc < L::KC; ++kc) {
                tc::tma_load_4d(smem + L::kOffK + st * L::kKVBytes + kc * L::kKVChunk, &tm_k, &bars->kv_full[st],
                                kc * 64, g, tok0, b);
                tc::tma_load_4d(smem + L::kOffV + st * L::kKVBytes + kc * L::kKVChunk, &tm_v, &bars->kv_full[st],
                                kc * 64, g, tok0, b);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          ++i;
        }
      }
    }
    if (lane == 0) {
      // let every issued copy land before the CTA can retire
      for (int j = (i > kStages ? i - kStages : 0); j < i; ++j)
        tc::mbar_wait(&bars->kv_full[j % kStages], (j / kStages) & 1);
    }
  } else if (warp == kMmaWarpR) {
    // ------------------------------------------------------------ MMA issuer
    auto wait_all = [&](uint64_t* bar, uint32_t par) { return __all_sync(0xffffffffu, tc::mbar_wait(bar, par)); };
    bool ok = wait_all(&bars->qo_full, 0);
    if (!ok) failr(bars, p.status, 51);
    tc::fence_after_sync();
    const uint64_t kdesc0 = tc::smem_desc_sw128(smem + L::kOffK, 16, 1024);
    const uint64_t vdesc0 = tc::smem_desc_sw128(smem + L::kOffV, 16, 1024);
    const uint64_t kdesc_mn0 = tc::smem_desc_sw128(smem + L::kOffK, L::kKVChunk, 1024);
    // dQ += dS K of step j (dS packed over S of buffer j & 1; K MN-major)
    auto issue_dq = [&](int j) -> bool {
      if (!wait_all(&bars->p_full[j & 1], (j >> 1) & 1)) return false;
      tc::fence_after_sync();
      const uint64_t kd = kdesc_mn0 + (uint64_t)(((j % kStages) * L::kKVBytes) >> 4);
      const uint32_t a_tm = tmem + L::kColSD + (j & 1) * 128;
#pragma unroll
      for (int k = 0; k < kStepR / 16; ++k)
        tc::mma_f16_ts_w(tmem + L::kColDQ, a_tm + k * 8, kd + (uint64_t)((k * 2048) >> 4), kIdescQ,
                         (j > 0 || k > 0) ? 1u : 0u);
      tc::mma_commit_w(&bars->kv_empty[j % kStages]);
      return true;
    };
    int i = 0;
    for (; ok && i < n_steps; ++i) {
      const int st = i % kStages;
      if (!wait_all(&bars->kv_full[st], (i / kStages) & 1)) {
        failr(bars, p.status, 52);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint64_t off = (uint64_t)((st * L::kKVBytes) >> 4);
      const uint32_t s_tm = tmem + L::kColSD + (i & 1) * 128;
      // S = Q K^T and dP = dout V^T over d, 16 at a time
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t ko = off + (uint64_t)((((k >> 2) * L::kKVChunk) + (k & 3) * 32) >> 4);
        tc::mma_f16_ts_w(s_tm, tmem + L::kColQ + k * 8, kdesc0 + ko, kIdescS, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t ko = off + (uint64_t)((((k >> 2) * L::kKVChunk) + (k & 3) * 32) >> 4);
        tc::mma_f16_ts_w(s_tm + 64, tmem + L::kColO + k * 8, vdesc0 + ko, kIdescS, k > 0 ? 1u : 0u);
      }
      tc::mma_commit_w(&bars->s_full[i & 1]);
      // the previous step's dQ, behind this step's S and dP on the tensor pipe
      if (i >= 1 && !issue_dq(i - 1)) {
        failr(bars, p.status, 53);
        ok = false;
        break;
      }
    }
    if (ok && i >= 1 && !issue_dq(i - 1)) failr(bars, p.status, 54);
    // dq_final completes once every MMA issued above has
    tc::mma_commit_w(&bars->dq_final);
    tc::mbar_wait(&bars->dq_final, 0);
  } else {
    // ------------------------------------------------------------ row threads (warps 0-3)
    const int r = threadIdx.x;  // tile row = TMEM lane
    const int pos = pos0 + r / G, hh = r % G, head = g * G + hh;
    const bool valid = pos < p.S;
    const int t = pos / p.block;
    const int n_blocks = (p.S + p.block - 1) / p.block;
    const int n_cand = p.causal ? t : n_blocks - 1;
    const float beta2 = n_cand > 0 ? p.sigma * logf(1.0f / (float)n_cand) * kLog2e : 0.f;
    const int64_t row = bg * p.S + (valid ? pos : 0);
    const int cnt = valid ? min(max(p.cnt[row], 0), (int)p.t_cap) : 0;
    const float* lp = p.logp + row * p.t_cap;
    const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);
    const float sc = rsqrtf((float)D) * kLog2e;
    const int64_t hrow = ((int64_t)b * p.H + head) * p.S + (valid ? pos : 0);
    const float lse2 = valid ? p.lse[hrow] : 0.f;
    float dd = 0.f;
    {
      // Q and dout rows into TMEM (the raw 16-bit pairs are the packed columns), D = dout . out
      const T* qs = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)(valid ? pos : 0) * p.q.ss +
                    (int64_t)head * p.q.sh;
      const T* ds = static_cast<const T*>(p.dout.data) + (int64_t)b * p.dout.sb +
                    (int64_t)(valid ? pos : 0) * p.dout.ss + (int64_t)head * p.dout.sh;
      const T* os = static_cast<const T*>(p.o.data) + (int64_t)b * p.o.sb + (int64_t)(valid ? pos : 0) * p.o.ss +
                    (int64_t)head * p.o.sh;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t wq[32], wo[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 xq = make_uint4(0u, 0u, 0u, 0u), xo = xq, xa = xq;
          if (valid) {
            xq = __ldg(reinterpret_cast<const uint4*>(qs + cc * 64 + v * 8));
            xo = __ldg(reinterpret_cast<const uint4*>(ds + cc * 64 + v * 8));
            xa = __ldg(reinterpret_cast<const uint4*>(os + cc * 64 + v * 8));
          }
          wq[4 * v] = xq.x, wq[4 * v + 1] = xq.y, wq[4 * v + 2] = xq.z, wq[4 * v + 3] = xq.w;
          wo[4 * v] = xo.x, wo[4 * v + 1] = xo.y, wo[4 * v + 2] = xo.z, wo[4 * v + 3] = xo.w;
          float fo[8], fa[8];
          Elt<T>::to_float(xo, fo);
          Elt<T>::to_float(xa, fa);
#pragma unroll
          for (int e = 0; e < 8; ++e) dd = fmaf(fo[e], fa[e], dd);
        }
        tc::tmem_st32(tbase + L::kColQ + cc * 32, wq);
        tc::tmem_st32(tbase + L::kColO + cc * 32, wo);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->qo_full);
      if (valid) p.dd[hrow] = dd;
    }
    // the row's list entries in order: entry `e_next` is the next block it selected
    int e_next = 0;
    int e_cur = -1;        // entry of the current block (-1: not selected, or the diagonal)
    float bias2 = kNegInf;  // bias of the current block, log2 units
    float dl = 0.f;         // sum of dS over the current block
    float* dz_row = p.dz + row * p.t_cap * G + hh;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      const int st = i % kStages;
      // the step's descriptor is published with its K/V copies
      if (!tc::mbar_wait(&bars->kv_full[st], (i / kStages) & 1)) {
        failr(bars, p.status, 55);
        ok = false;
        break;
      }
      const StepR d = bars->desc[st];
      if (d.first) {
        e_cur = -1;
        bias2 = kNegInf;
        dl = 0.f;
        if (valid) {
          if (d.c == t) {
            bias2 = beta2;
          } else {
            const uint32_t w = r / G < 32 ? d.mask.x : r / G < 64 ? d.mask.y : r / G < 96 ? d.mask.z : d.mask.w;
            if (((w >> ((r / G) & 31)) & 1u) && e_next < cnt) {
              e_cur = e_next++;
              bias2 = p.sigma * __ldg(lp + e_cur) * kLog2e;
            }
          }
        }
      }
      const int sb = i & 1;
      if (!tc::mbar_wait(&bars->s_full[sb], (i >> 1) & 1)) {
        failr(bars, p.status, 56);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      // keys of this step the row sees: none if it did not select the block,
      // fewer on the causal diagonal and at the ragged end
      int n_valid = bias2 == kNegInf ? 0 : kStepR;
      if (d.tok0 + kStepR > p.S) n_valid = min(n_valid, p.S - d.tok0);
      if (p.causal && d.c == t) n_valid = min(n_valid, pos - d.tok0 + 1);
      const float off = bias2 - lse2;
      const uint32_t s_tm = tbase + L::kColSD + sb * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t sv[32], pv[32], dw[16];
        tc::tmem_ld32(s_tm + ch * 32, sv);
        tc::tmem_ld32(s_tm + 64 + ch * 32, pv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float dsv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key = ch * 32 + j + u;
            const float pr = key < n_valid ? tc::ex2(fmaf(__uint_as_float(sv[j + u]), sc, off)) : 0.f;
            dsv[u] = pr * (__uint_as_float(pv[j + u]) - dd);
            dl += dsv[u];
          }
          dw[j >> 1] = pack2<T>(dsv[0], dsv[1]);
        }
        tc::tmem_st16(s_tm + ch * 16, dw);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full[sb]);
      if (d.last && e_cur >= 0) dz_row[(int64_t)e_cur * G] = p.sigma * dl;
    }
    // ---- epilogue: dq = dQ / sqrt(d)
    if (ok && tc::mbar_wait(&bars->dq_final, 0)) {
      tc::fence_after_sync();
      const float qsc = rsqrtf((float)D);
      float* dqg = static_cast<float*>(const_cast<void*>(p.dq.data)) + (int64_t)b * p.dq.sb +
                   (int64_t)(valid ? pos : 0) * p.dq.ss + (int64_t)head * p.dq.sh;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tc::tmem_ld32(tbase + L::kColDQ + cc * 32, v);
        tc::tmem_wait_ld();
        if (n_steps == 0) {
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(dqg + cc * 32 + q * 4) =
                make_float4(__uint_as_float(v[q * 4]) * qsc, __uint_as_float(v[q * 4 + 1]) * qsc,
                            __uint_as_float(v[q * 4 + 2]) * qsc, __uint_as_float(v[q * 4 + 3]) * qsc);
        }
      }
    } else if (ok) {
      failr(bars, p.status, 57);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarpR) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <typename T, int D>
cudaError_t launch_row_tc(const BwdParams& p, cudaStream_t stream) {
  using L = RowLayout<D>;
  CUtensorMap mk, mv;
  if (!make_map(&mk, p.k, p.dtype, p.B, p.S, p.Hkv, D, 1, kStepR) ||
      !make_map(&mv, p.v, p.dtype, p.B, p.S, p.Hkv, D, 1, kStepR))
    return cudaErrorInvalidValue;
  auto kern = bwd_row_tc_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.n_tiles, p.Hkv, p.B), kThreadsR, L::kAlloc, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_row_tc(const BwdParams& p, cudaStream_t stream) {
  if (p.dtype == 1) return p.D == 128 ? launch_row_tc<__half, 128>(p, stream) : launch_row_tc<__half, 64>(p, stream);
  return p.D == 128 ? launch_row_tc<__nv_bfloat16, 128>(p, stream) : launch_row_tc<__nv_bfloat16, 64>(p, stream);
}

}  // namespace dash
