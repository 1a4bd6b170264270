// Stage 2 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: softmax(l + log g) over the tokens of the selected blocks, g = 0
// (masked) on blocks without routing mass, the near-diagonal block always
// included; the pages' kernel walks the active chunks of a FlashAttention
// loop and adds the routing bias before the softmax.
//
// A tile is 128 rows = (128 / G positions) x (G heads of one KV group), so
// each K/V block brought in serves every head of the group.  One CTA owns two
// adjacent tiles and walks the ascending work list of the pair (the union of
// both tiles' lists, each block with the mask of positions per tile that
// selected it) in 64-token steps; while the softmax of one tile runs, the
// tensor core works on the other's products.
//
// Tensor memory holds, per tile, the query rows (the A operand of S = Q K^T),
// S, and O; P is written back over S (bf16/f16, two per column) and is the A
// operand of O += P V.  Shared memory then only carries the K/V ring, so each
// step reads 16 KB of K and 16 KB of V from it per tile.  Warp roles:
//   warp 8      TMA producer: K and V of each step into a ring of stages
//               (128-byte swizzle, the layout the MMA reads), publishing the
//               step's block, first token and masks.
//   warp 9      MMA issuer (one thread) and TMEM owner.  Per step and tile,
//               in this order: O += P V of the previous step, then S = Q K^T
//               of this step (in-order execution lets S overwrite P).
//   warps 0-3   softmax of tile 0, warps 4-7 of tile 1: thread r owns row r
//               (= TMEM lane r).  It first stores its query row into TMEM,
//               then per step reads its 64 logits, adds the row's prior bias
//               (log p_bar of the block if its position selected it,
//               log(1/N) on its own block, else -inf), keeps the running max
//               and sum, writes P into TMEM and finally normalises O.  P is
//               taken against the row's reference max; the step's row max is
//               only computed when the row has no reference yet or the step's
//               sum shows a P above 2^8.  O is rescaled in TMEM only when the
//               reference grows by more than 2^8, so P stays <= 256 and the
//               result is exact (the final division uses the same reference).
//               The scale-and-offset FMAs and the row sums use paired fp32
//               instructions.
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
constexpr int kTiles = 2;
constexpr int kStep = 64;                   // tokens per step
constexpr int kMaxStages = 8;               // bound of the K/V ring depth
constexpr int kProducerWarp = 4 * kTiles;   // warp 8
constexpr int kMmaWarp = kProducerWarp + 1; // warp 9
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kTmemCols = 512;
// TMEM columns of tile t: Q at 256 t (D / 2 columns), S (and P over it) at
// 256 t + 64, O at 256 t + 128 (D columns)
constexpr int kTileCols = 256;
constexpr int kSOff = 64;
constexpr int kOOff = 128;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Layout {
  static constexpr int KC = D / 64;               // 128-byte chunks of a row
  static constexpr int kKVChunk = kStep * 128;    // 8 KB
  static constexpr int kKVBytes = KC * kKVChunk;  // one K (or V) stage
  static constexpr int kStages = D == 128 ? 6 : 8;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  static constexpr int kBytes = kOffBar + 768;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// What the producer tells the other roles about a step (one per ring stage).
struct StepDesc {
  int c, tok0, first, pad;
  uint4 mask[kTiles];
};

struct Bars {
  uint64_t q_full;  // query rows stored into TMEM (256 arrivals)
  uint64_t kv_full[kMaxStages];
  uint64_t kv_empty[kMaxStages];
  uint64_t s_full[kTiles];
  uint64_t p_full[kTiles];
  uint64_t o_final;
  uint32_t tmem_base;
  int abort;
  StepDesc desc[kMaxStages];
};

__device__ __forceinline__ void fail_timeout(Bars* bars, DeviceStatus* st, int where) {
  raise_status(st, 5 /* DASH_ERR_DEVICE_TIMEOUT */, where);
  atomicExch(&bars->abort, 1);
}


template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             SparseParams p) {
  using L = Layout<D>;
  constexpr int kStages = L::kStages;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = tc::idesc_f16(kRows, kStep, kBF16, false, false);
  constexpr uint32_t kIdescO = tc::idesc_f16(kRows, D, kBF16, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, g = blockIdx.y, pair = blockIdx.x;
  const int G = p.G;
  const int P = p.tile_pos;  // 128 / G positions per tile
  const int pos0 = pair * kTiles * P;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int64_t pix = bg * p.n_pairs + pair;
  const int32_t* plist = p.plist + pix * p.t_cap;
  const uint4* pmask = p.pmask + pix * p.t_cap * kTiles;
  const int pcnt = p.pcnt[pix];
  const int n_steps = p.psteps[pix];
  // how long a consumer waits for a hand-off (drains keep the default)
  const long long budget = p.wait_cycles > 0 ? p.wait_cycles : tc::kWaitCycles;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, kTiles * kRows);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
    }
    for (int t = 0; t < kTiles; ++t) {
      tc::mbar_init(&bars->s_full[t], 1);
      tc::mbar_init(&bars->p_full[t], kRows);
    }
    tc::mbar_init(&bars->o_final, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&bars->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tc::prefetch_tensormap(&tm_k);
    tc::prefetch_tensormap(&tm_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the pair's work list 32 entries at a time (one
    // coalesced load per lane); lane 0 issues the copies.
    const int spb = p.block / kStep;
    const int last_needed = p.causal ? min(pos0 + kTiles * P, p.S) - 1 : p.S - 1;
    int i = 0;
    bool ok = true;
    for (int u0 = 0; ok && !p.stall_producer && u0 < pcnt; u0 += 32) {
      const bool have = u0 + lane < pcnt;
      const int my_c = have ? __ldg(plist + u0 + lane) : 0;
      const uint4 my_m0 = have ? __ldg(pmask + (u0 + lane) * kTiles) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 my_m1 = have ? __ldg(pmask + (u0 + lane) * kTiles + 1) : make_uint4(0u, 0u, 0u, 0u);
      const int nj = min(32, pcnt - u0);
      for (int j = 0; ok && j < nj; ++j) {
        const int c = __shfl_sync(0xffffffffu, my_c, j);
        uint4 m0, m1;
        m0.x = __shfl_sync(0xffffffffu, my_m0.x, j);
        m0.y = __shfl_sync(0xffffffffu, my_m0.y, j);
        m0.z = __shfl_sync(0xffffffffu, my_m0.z, j);
        m0.w = __shfl_sync(0xffffffffu, my_m0.w, j);
        m1.x = __shfl_sync(0xffffffffu, my_m1.x, j);
        m1.y = __shfl_sync(0xffffffffu, my_m1.y, j);
        m1.z = __shfl_sync(0xffffffffu, my_m1.z, j);
        m1.w = __shfl_sync(0xffffffffu, my_m1.w, j);
        for (int h = 0; h < spb; ++h) {
          const int tok0 = c * p.block + h * kStep;
          if (tok0 > last_needed) continue;
          if (lane == 0) {
            const int st = i % kStages;
            if (i >= kStages && !tc::mbar_wait(&bars->kv_empty[st], ((i / kStages) - 1) & 1, budget)) {
              fail_timeout(bars, p.status, 1);
              ok = false;
            } else {
              StepDesc& d = bars->desc[st];
              d.c = c;
              d.tok0 = tok0;
              d.first = h == 0;
              d.mask[0] = m0;
              d.mask[1] = m1;
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
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (descriptors stay warp-uniform);
    // one elected lane issues each MMA and commit.
    auto wait_all = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, par, budget));
    };
    bool ok = wait_all(&bars->q_full, 0);
    if (!ok) fail_timeout(bars, p.status, 2);
    tc::fence_after_sync();
    // Descriptors of stage 0; a stage or k-slice offset only moves the start
    // address field (bytes >> 4), so the issue loops add constants.
    const uint64_t kdesc0 = tc::smem_desc_sw128(smem + L::kOffK, 16, 1024);
    const uint64_t vdesc0 = tc::smem_desc_sw128(smem + L::kOffV, L::kKVChunk, 1024);
    // O(t) += P(t) V of step j, A = P from TMEM (over S)
    auto issue_pv = [&](int t, int j) -> bool {
      if (!wait_all(&bars->p_full[t], j & 1)) return false;
      tc::fence_after_sync();
      const uint64_t vd = vdesc0 + (uint64_t)(((j % kStages) * L::kKVBytes) >> 4);
      const uint32_t d_tm = tmem + t * kTileCols + kOOff, a_tm = tmem + t * kTileCols + kSOff;
      tc::mma_f16_ts_w(d_tm, a_tm, vd, kIdescO, j > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 1; k < kStep / 16; ++k) tc::mma_f16_ts_w(d_tm, a_tm + k * 8, vd + ((k * 2048) >> 4), kIdescO, 1u);
      return true;
    };
    int i = 0;
    for (; ok && i < n_steps; ++i) {
      const int st = i % kStages;
      if (!wait_all(&bars->kv_full[st], (i / kStages) & 1)) {
        fail_timeout(bars, p.status, 3);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      for (int t = 0; ok && t < kTiles; ++t) {
        if (i >= 1 && !issue_pv(t, i - 1)) {
          fail_timeout(bars, p.status, 4);
          ok = false;
          break;
        }
        // S(t) = Q(t) K^T, A = Q from TMEM
        const uint64_t kd = kdesc0 + (uint64_t)((st * L::kKVBytes) >> 4);
        const uint32_t s_tm = tmem + t * kTileCols + kSOff, q_tm = tmem + t * kTileCols;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_f16_ts_w(s_tm, q_tm + k * 8, kd + (uint64_t)((((k >> 2) * L::kKVChunk) + (k & 3) * 32) >> 4),
                           kIdescS, k > 0 ? 1u : 0u);
        tc::mma_commit_w(&bars->s_full[t]);
      }
      if (ok && i >= 1) tc::mma_commit_w(&bars->kv_empty[(i - 1) % kStages]);
    }
    if (ok && i >= 1) {
      for (int t = 0; ok && t < kTiles; ++t)
        if (!issue_pv(t, i - 1)) {
          fail_timeout(bars, p.status, 5);
          ok = false;
        }
    }
    // o_final arrives once every MMA issued above has completed
    tc::mma_commit_w(&bars->o_final);
    tc::mbar_wait(&bars->o_final, 0);
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int t = warp >> 2;  // tile
    const int q4 = warp & 3;  // TMEM lane quarter
    const int r = q4 * 32 + lane;
    RowPrior row;
    if (p.logp_dense)
      row.init_dense(p, bg, pos0 + t * P + r / G, r / G, plist, pcnt);
    else
      row.init(p, bg, pos0 + t * P + r / G, r / G);
    const int head = g * G + r % G;
    const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + t * kTileCols;
    const float qk_scale = rsqrtf((float)D) * kLog2e;
    {
      // the query row into TMEM: the raw 16-bit pairs are the packed columns
      const T* src = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb +
                     (int64_t)(row.valid ? row.pos : 0) * p.q.ss + (int64_t)head * p.q.sh;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (row.valid) x = __ldg(reinterpret_cast<const uint4*>(src + cc * 64 + v * 8));
          w[4 * v] = x.x;
          w[4 * v + 1] = x.y;
          w[4 * v + 2] = x.z;
          w[4 * v + 3] = x.w;
        }
        tc::tmem_st32(tbase + cc * 32, w);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->q_full);
    }
    float m_used = kNegInf, lsum = 0.f, bias = kNegInf;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      const int st = i % kStages;
      // the step's descriptor is published with its K/V copies
      if (!tc::mbar_wait(&bars->kv_full[st], (i / kStages) & 1, budget)) {
        fail_timeout(bars, p.status, 10);
        ok = false;
        break;
      }
      const int c = bars->desc[st].c, tok0 = bars->desc[st].tok0;
      if (bars->desc[st].first) bias = row.bias(c, bars->desc[st].mask[t]);
      if (!tc::mbar_wait(&bars->s_full[t], i & 1, budget)) {
        fail_timeout(bars, p.status, 6);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sv[kStep];
      tc::tmem_ld32(tbase + kSOff, sv);
      tc::tmem_ld32(tbase + kSOff + 32, sv + 32);
      tc::tmem_wait_ld();

      // valid columns of this row in this step: 0 when the row did not select
      // the block, fewer on the causal diagonal and at the ragged end
      int n_valid = bias == kNegInf ? 0 : kStep;
      if (tok0 + kStep > p.S) n_valid = min(n_valid, p.S - tok0);
      if (p.causal && c == row.t) n_valid = min(n_valid, row.pos - tok0 + 1);
      const float b2 = bias * kLog2e;
      // masked columns hold -inf and give p = 0
      if (n_valid < kStep) {
#pragma unroll
        for (int j = 0; j < kStep; ++j)
          if (j >= n_valid) sv[j] = __float_as_uint(kNegInf);
      }
      uint32_t pw[32];
      // p = 2^(s * scale + bias - m) for the 64 columns; returns their sum
      auto exps = [&](float off) -> float {
        const float2 sc2 = make_float2(qk_scale, qk_scale), off2 = make_float2(off, off);
        float2 ps2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) ps2[e] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kStep; j += 2) {
          const float2 a = __ffma2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), sc2, off2);
          const float2 pp = make_float2(tc::ex2(a.x), tc::ex2(a.y));
          ps2[(j >> 1) & 3] = __fadd2_rn(ps2[(j >> 1) & 3], pp);
          pw[j >> 1] = pack2<T>(pp.x, pp.y);
        }
        const float2 s01 = __fadd2_rn(__fadd2_rn(ps2[0], ps2[1]), __fadd2_rn(ps2[2], ps2[3]));
        return s01.x + s01.y;
      };
      // Fast path: the row's running reference max m_used is kept; valid
      // while every p stays <= 2^8, which the step's sum bounds.  Otherwise
      // (no reference yet, or a larger max) the row max is taken and the
      // step recomputed; O is rescaled when the reference grows by > 2^8.
      float corr = 1.0f;
      bool resc = false;
      const bool fast = m_used != kNegInf && n_valid > 0;
      float lstep = fast ? exps(b2 - m_used) : 0.f;
      if (!fast || !(lstep <= 256.0f)) {
        // the bias is constant over the step and the scale positive, so the
        // row max of the logits is max(s) * scale + bias
        float pm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = __uint_as_float(sv[e]);
#pragma unroll
        for (int j = 8; j < kStep; ++j) pm[j & 7] = fmaxf(pm[j & 7], __uint_as_float(sv[j]));
        const float smax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float mx = n_valid > 0 ? fmaf(smax, qk_scale, b2) : kNegInf;
        if (mx != kNegInf) {
          if (m_used == kNegInf) {
            m_used = mx;  // nothing accumulated for this row yet
          } else if (mx > m_used + kRescaleLog2) {
            corr = tc::ex2(m_used - mx);
            m_used = mx;
            resc = true;
          }
        }
        lstep = exps(n_valid > 0 ? b2 - m_used : kNegInf);
      }
      lsum = lsum * corr + lstep;
      tc::tmem_st32(tbase + kSOff, pw);
      if (__any_sync(0xffffffffu, resc)) {
        // O rescaled to the new reference before this step's P V is issued;
        // O is stable: the previous step's P V completed before this S
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          const uint32_t ta = tbase + kOOff + cc * 32;
          tc::tmem_ld32(ta, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * corr);
          tc::tmem_st32(ta, ov);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full[t]);
    }
    // ---- epilogue: the row's log-sum-exp (log2 units) if wanted, O / l -> out
    if (ok && p.lse && row.valid) p.lse[((int64_t)b * p.H + head) * p.S + row.pos] = m_used + log2f(lsum);
    if (p.skip_out) {
      // nothing to read back; the MMA warp drains its MMAs before TMEM is freed
    } else if (ok && tc::mbar_wait(&bars->o_final, 0, budget)) {
      tc::fence_after_sync();
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      T* dst = static_cast<T*>(const_cast<void*>(p.out.data)) + (int64_t)b * p.out.sb +
               (int64_t)(row.valid ? row.pos : 0) * p.out.ss + (int64_t)head * p.out.sh;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tc::tmem_ld32(tbase + kOOff + cc * 32, ov);
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
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

namespace {
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

}  // namespace

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

namespace {

template <typename T, int D>
cudaError_t launch_tc(const SparseParams& p, cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!make_map(&mk, p.k, p.dtype, p.B, p.S, p.Hkv, D, 1, kStep) ||
      !make_map(&mv, p.v, p.dtype, p.B, p.S, p.Hkv, D, 1, kStep))
    return cudaErrorInvalidValue;
  using L = Layout<D>;
  auto kern = sparse_prefill_tc_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_pairs, p.Hkv, p.B);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

int sparse_tile_pair() { return kTiles; }

cudaError_t launch_sparse_prefill_tc(const SparseParams& p, cudaStream_t stream) {
  if (p.D == 128) {
    if (p.dtype == 1) return launch_tc<__half, 128>(p, stream);
    return launch_tc<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 1) return launch_tc<__half, 64>(p, stream);
  return launch_tc<__nv_bfloat16, 64>(p, stream);
}

}  // namespace dash
