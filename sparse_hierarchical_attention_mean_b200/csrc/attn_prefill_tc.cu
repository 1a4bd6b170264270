// Stage 2 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: softmax(l + log g) over the tokens of the selected blocks, g = 0
// (masked) on blocks without routing mass, the near-diagonal block always
// included; the pages' kernel walks the active chunks of a FlashAttention
// loop and adds the routing bias before the softmax.
//
// One CTA owns a tile of 128 rows = (128 / G positions) x (G heads of one KV
// group), so each K/V block brought in serves every head of the group.  It
// walks the tile's ascending work list (the union of its rows' selected
// blocks plus the rows' own blocks) in 64-token steps.  Warp roles:
//   warp 4      TMA producer: Q once, then K and V of each step into a
//               3-stage ring (128-byte swizzle, the layout the MMA reads).
//   warp 5      MMA issuer (one thread) and TMEM owner: S = Q K^T into one of
//               two 64-column TMEM buffers, then O += P V into 128 TMEM
//               columns once the softmax has written P.
//   warps 0-3   softmax: thread r owns row r (= TMEM lane r).  It reads its
//               64 logits from TMEM, adds its own prior bias (walking its own
//               ascending block list), keeps the running max and sum, writes
//               P (bf16/f16) to shared memory for the next MMA and finally
//               normalises O.  O is rescaled in TMEM only when a row's max
//               grows by more than 2^8, so P stays <= 256 and the result is
//               exact (the final division uses the same reference max).
// Every mbarrier wait is bounded; on expiry the kernel records
// DASH_ERR_DEVICE_TIMEOUT in the workspace status word and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "sparse_common.cuh"
#include "tc.cuh"

namespace dash {
namespace {

constexpr int kRows = 128;
constexpr int kStep = 64;      // tokens per step
constexpr int kStages = 3;     // K/V ring depth
constexpr int kThreads = 192;  // 4 softmax warps + producer + MMA
constexpr int kTmemCols = 256;
constexpr int kSCol = 0;    // two S buffers of 64 fp32 columns
constexpr int kOCol = 128;  // O accumulator (D columns)
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Layout {
  static constexpr int KC = D / 64;               // 128-byte chunks of a row
  static constexpr int kQChunk = kRows * 128;     // 16 KB
  static constexpr int kKVChunk = kStep * 128;    // 8 KB
  static constexpr int kKVBytes = KC * kKVChunk;  // one K (or V) stage
  static constexpr int kPBytes = kRows * 128;     // 128 rows x 64 16-bit values
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + KC * kQChunk;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffP = kOffV + kStages * kKVBytes;
  static constexpr int kOffBar = kOffP + 2 * kPBytes;
  static constexpr int kBytes = kOffBar + 512;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// What the producer tells the softmax warps about a step (one per ring stage).
struct StepDesc {
  int c, tok0, first, pad;
  uint4 mask;
};

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t o_final;
  uint32_t tmem_base;
  int abort;
  StepDesc desc[kStages];
};

__device__ __forceinline__ void fail_timeout(Bars* bars, DeviceStatus* st, int where) {
  raise_status(st, 5 /* DASH_ERR_DEVICE_TIMEOUT */, where);
  atomicExch(&bars->abort, 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, SparseParams p) {
  using L = Layout<D>;
  constexpr bool kBF16 = sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = tc::idesc_f16(kRows, kStep, kBF16, false, false);
  constexpr uint32_t kIdescO = tc::idesc_f16(kRows, D, kBF16, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y, tile = blockIdx.x;
  const int G = p.G;
  const int P = p.tile_pos;  // 128 / G
  const int pos0 = tile * P;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int32_t* ulist = p.ulist + (bg * p.n_tiles + tile) * p.t_cap;
  const int ucnt = p.ucnt[bg * p.n_tiles + tile];
  const int n_steps = p.usteps[bg * p.n_tiles + tile];
  const int last_pos = min(pos0 + P, p.S) - 1;
  const int last_needed = p.causal ? last_pos : p.S - 1;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->s_free[s], 128);
      tc::mbar_init(&bars->p_full[s], 128);
      tc::mbar_init(&bars->pv_done[s], 1);
    }
    tc::mbar_init(&bars->o_final, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(&bars->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tensormap(&tm_q);
    tc::prefetch_tensormap(&tm_k);
    tc::prefetch_tensormap(&tm_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the work list 32 entries at a time (one coalesced
    // load per lane); lane 0 issues the copies.
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(&bars->q_full, L::KC * L::kQChunk);
      for (int kc = 0; kc < L::KC; ++kc)
        tc::tma_load_4d(smem + L::kOffQ + kc * L::kQChunk, &tm_q, &bars->q_full, kc * 64, g * G, pos0, b);
    }
    const uint4* umask = p.umask + (bg * p.n_tiles + tile) * p.t_cap;
    const int spb = p.block / kStep;
    int i = 0;
    bool ok = true;
    for (int u0 = 0; ok && u0 < ucnt; u0 += 32) {
      const int my_c = u0 + lane < ucnt ? __ldg(ulist + u0 + lane) : 0;
      const uint4 my_m = u0 + lane < ucnt ? __ldg(umask + u0 + lane) : make_uint4(0u, 0u, 0u, 0u);
      const int nj = min(32, ucnt - u0);
      for (int j = 0; ok && j < nj; ++j) {
        const int c = __shfl_sync(0xffffffffu, my_c, j);
        uint4 m;
        m.x = __shfl_sync(0xffffffffu, my_m.x, j);
        m.y = __shfl_sync(0xffffffffu, my_m.y, j);
        m.z = __shfl_sync(0xffffffffu, my_m.z, j);
        m.w = __shfl_sync(0xffffffffu, my_m.w, j);
        for (int h = 0; h < spb; ++h) {
          const int tok0 = c * p.block + h * kStep;
          if (tok0 > last_needed) continue;
          if (lane == 0) {
            const int st = i % kStages;
            if (i >= kStages && !tc::mbar_wait(&bars->kv_empty[st], ((i / kStages) - 1) & 1)) {
              fail_timeout(bars, p.status, 1);
              ok = false;
            } else {
              StepDesc& d = bars->desc[st];
              d.c = c;
              d.tok0 = tok0;
              d.first = h == 0;
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
      tc::mbar_wait(&bars->q_full, 0);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = tc::mbar_wait(&bars->q_full, 0);
      if (!ok) fail_timeout(bars, p.status, 2);
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1, st = j % kStages;
        if (!tc::mbar_wait(&bars->p_full[pb], (j >> 1) & 1)) return false;
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < kStep / 16; ++k) {
          const uint64_t ad = tc::smem_desc_sw128(smem + L::kOffP + pb * L::kPBytes + k * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(smem + L::kOffV + st * L::kKVBytes + k * 2048, L::kKVChunk, 1024);
          tc::mma_f16_ss(tmem + kOCol, ad, bd, kIdescO, (j > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(&bars->pv_done[pb]);
        tc::mma_commit(&bars->kv_empty[st]);
        return true;
      };
      int i = 0;
      for (; ok && i < n_steps; ++i) {
        const int st = i % kStages, sb = i & 1;
        if (!tc::mbar_wait(&bars->kv_full[st], (i / kStages) & 1) ||
            (i >= 2 && !tc::mbar_wait(&bars->s_free[sb], ((i >> 1) - 1) & 1))) {
          fail_timeout(bars, p.status, 3);
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t ad = tc::smem_desc_sw128(smem + L::kOffQ + (k >> 2) * L::kQChunk + (k & 3) * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(
              smem + L::kOffK + st * L::kKVBytes + (k >> 2) * L::kKVChunk + (k & 3) * 32, 16, 1024);
          tc::mma_f16_ss(tmem + kSCol + sb * kStep, ad, bd, kIdescS, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->s_full[sb]);
        if (i >= 1 && !issue_pv(i - 1)) {
          fail_timeout(bars, p.status, 4);
          ok = false;
          break;
        }
      }
      if (ok && i >= 1 && !issue_pv(i - 1)) fail_timeout(bars, p.status, 5);
      // o_final arrives once every MMA issued above has completed
      tc::mma_commit(&bars->o_final);
      tc::mbar_wait(&bars->o_final, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int r = threadIdx.x;
    RowPrior row;
    row.init(p, bg, pos0 + r / G, r / G);
    const int head = g * G + r % G;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float qk_scale = rsqrtf((float)D) * kLog2e;
    uint8_t* prow = smem + L::kOffP + r * 128;
    float m_used = kNegInf, lsum = 0.f, bias = kNegInf;
    bool ok = true;
    int i = 0;
    for (; i < n_steps; ++i) {
      const int sb = i & 1, st = i % kStages;
      // the step's descriptor is published with its K/V copies
      if (!tc::mbar_wait(&bars->kv_full[st], (i / kStages) & 1)) {
        fail_timeout(bars, p.status, 10);
        ok = false;
        break;
      }
      const int c = bars->desc[st].c, tok0 = bars->desc[st].tok0;
      if (bars->desc[st].first) bias = row.bias(c, bars->desc[st].mask);
      if (!tc::mbar_wait(&bars->s_full[sb], (i >> 1) & 1)) {
        fail_timeout(bars, p.status, 6);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sv[kStep];
      tc::tmem_ld32(tmem + lane_base + kSCol + sb * kStep, sv);
      tc::tmem_ld32(tmem + lane_base + kSCol + sb * kStep + 32, sv + 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->s_free[sb]);

      // valid columns of this row in this step: 0 when the row did not select
      // the block, fewer on the causal diagonal and at the ragged end
      int n_valid = bias == kNegInf ? 0 : kStep;
      if (tok0 + kStep > p.S) n_valid = min(n_valid, p.S - tok0);
      if (p.causal && c == row.t) n_valid = min(n_valid, row.pos - tok0 + 1);
      const float b2 = bias * kLog2e;
      if (n_valid == kStep) {
#pragma unroll
        for (int j = 0; j < kStep; ++j) sv[j] = __float_as_uint(fmaf(__uint_as_float(sv[j]), qk_scale, b2));
      } else {
#pragma unroll
        for (int j = 0; j < kStep; ++j)
          sv[j] = __float_as_uint(j < n_valid ? fmaf(__uint_as_float(sv[j]), qk_scale, b2) : kNegInf);
      }
      // row max: a tree over 8 independent partial maxima
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = __uint_as_float(sv[e]);
#pragma unroll
      for (int j = 8; j < kStep; ++j) pm[j & 7] = fmaxf(pm[j & 7], __uint_as_float(sv[j]));
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                             fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      float corr = 1.0f;
      bool resc = false;
      if (mx != kNegInf) {
        if (m_used == kNegInf) {
          m_used = mx;  // nothing accumulated for this row yet
        } else if (mx > m_used + kRescaleLog2) {
          corr = tc::ex2(m_used - mx);
          m_used = mx;
          resc = true;
        }
      }
      // P buffer sb is free once PV of step i-2 has completed
      if (i >= 2 && !tc::mbar_wait(&bars->pv_done[sb], ((i >> 1) - 1) & 1)) {
        fail_timeout(bars, p.status, 7);
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O is stable once PV of step i-1 has completed
        if (i >= 1 && !tc::mbar_wait(&bars->pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1)) {
          fail_timeout(bars, p.status, 8);
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tc::tmem_ld32(tmem + lane_base + kOCol + cc * 32, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * corr);
          tc::tmem_st32(tmem + lane_base + kOCol + cc * 32, ov);
        }
        tc::tmem_wait_st();
        lsum *= corr;
      }
      // masked entries are -inf and give 2^-inf = 0; a row with nothing
      // accumulated yet (m_used = -inf) writes zeros
      const float msub = m_used == kNegInf ? 0.f : m_used;
      uint8_t* pdst = prow + sb * L::kPBytes;
      float ps[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ps[e] = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = tc::ex2(__uint_as_float(sv[q * 8 + e]) - msub);
          ps[e] += pv[e];
        }
        uint4 w;
        w.x = pack2<T>(pv[0], pv[1]);
        w.y = pack2<T>(pv[2], pv[3]);
        w.z = pack2<T>(pv[4], pv[5]);
        w.w = pack2<T>(pv[6], pv[7]);
        *reinterpret_cast<uint4*>(pdst + ((q ^ (r & 7)) << 4)) = w;
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full[sb]);
    }
    // ---- epilogue: O / l -> out
    if (ok && tc::mbar_wait(&bars->o_final, 0)) {
      tc::fence_after_sync();
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      T* dst = static_cast<T*>(const_cast<void*>(p.out.data)) + (int64_t)b * p.out.sb +
               (int64_t)(row.valid ? row.pos : 0) * p.out.ss + (int64_t)head * p.out.sh;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tc::tmem_ld32(tmem + lane_base + kOCol + cc * 32, ov);
        tc::tmem_wait_ld();
        if (row.valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack2<T>(__uint_as_float(ov[q * 8 + 0]) * inv, __uint_as_float(ov[q * 8 + 1]) * inv);
            w.y = pack2<T>(__uint_as_float(ov[q * 8 + 2]) * inv, __uint_as_float(ov[q * 8 + 3]) * inv);
            w.z = pack2<T>(__uint_as_float(ov[q * 8 + 4]) * inv, __uint_as_float(ov[q * 8 + 5]) * inv);
            w.w = pack2<T>(__uint_as_float(ov[q * 8 + 6]) * inv, __uint_as_float(ov[q * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + cc * 32 + q * 8) = w;
          }
        }
      }
    } else if (ok) {
      fail_timeout(bars, p.status, 9);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D map over a [B, S, H, D] view (innermost first: D, H, S, B), 128-byte
// swizzle, box {64, box_h, box_s, 1}.
bool make_map(CUtensorMap* map, const View& v, int dtype, int64_t B, int64_t S, int64_t H, int D, int box_h,
              int box_s) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = 2;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(v.sh * es), (cuuint64_t)(v.ss * es),
                           (cuuint64_t)((B > 1 ? v.sb : S * v.ss) * es)};
  cuuint32_t box[4] = {64, (cuuint32_t)box_h, (cuuint32_t)box_s, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 4, const_cast<void*>(v.data), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T, int D>
cudaError_t launch_tc(const SparseParams& p, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, p.q, p.dtype, p.B, p.S, p.H, D, p.G, p.tile_pos) ||
      !make_map(&mk, p.k, p.dtype, p.B, p.S, p.Hkv, D, 1, kStep) ||
      !make_map(&mv, p.v, p.dtype, p.B, p.S, p.Hkv, D, 1, kStep))
    return cudaErrorInvalidValue;
  using L = Layout<D>;
  auto kern = sparse_prefill_tc_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_tiles, p.Hkv, p.B);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_prefill_tc(const SparseParams& p, cudaStream_t stream) {
  if (p.D == 128) {
    if (p.dtype == 1) return launch_tc<__half, 128>(p, stream);
    return launch_tc<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 1) return launch_tc<__half, 64>(p, stream);
  return launch_tc<__nv_bfloat16, 64>(p, stream);
}

}  // namespace dash
