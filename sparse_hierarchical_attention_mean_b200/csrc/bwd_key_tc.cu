// Key-centric backward on the 5th-generation tensor cores: dk, dv, the
// summary gradient and its stage-0 term.
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: a key of block c receives gradient from every query row that
// attends to it, i.e. the rows that selected c (bias sigma * log p_bar_c) and
// the rows whose own block c is (bias sigma * log(1/N), causal mask).
// "Stage 0: local chunk summary" and "Stage 1: entmax chunk routing": the
// summary s_c = mean(k) W_s also carries the routing gradient back, ds_c =
// gamma sum_rows dL/dz q, which reaches every key of c as ds_c W_s^T / |c|.
//
// One CTA owns 128 keys (two blocks of 64 or one of 128) of one KV head and
// walks, in order, the stage-2 tiles (128 rows: 128 / G positions x G heads)
// whose work list holds one of its blocks.  Per tile, with the tile's Q and
// dout rows brought in by TMA (4-D maps, 128-byte swizzle, no multicast):
//   S^T  = K Q^T     (SS MMA, M = 128 keys, N = 128 rows)    -> TMEM [0, 128)
//   dP^T = V dout^T  (SS MMA)                                -> TMEM [128, 256)
//   P^T  = 2^(S^T scale + bias_row - lse_row), dS^T = P^T (dP^T - D_row),
//          written back as bf16/f16 over S^T and dP^T (one thread per key)
//   dV  += P^T dout  (TS MMA, A = P^T from TMEM, dout MN-major) TMEM [256, 256 + d)
//   dK  += dS^T Q    (TS MMA, A = dS^T from TMEM, Q MN-major)   TMEM [384, 384 + d)
// Each row's log-sum-exp comes from the forward's stage-2 kernel, D = dout .
// out and the routing gradient dL/dz from the earlier backward kernels.
// Warps 0-7 own the keys (two per TMEM lane quarter, each taking half of the
// tile's rows); warps 8-11 prepare each tile's row data (D, and per block of
// the CTA the bias minus the log-sum-exp, the causal key limit and dL/dz: the
// block's position in the row's list is the row's count of selections in the
// words below plus a population count within the word) and then sum the summary gradient over the rows with dL/dz != 0
// from the Q tile in shared memory; warp 12 finds the tiles (bit masks of the
// tiles' work lists) and issues the copies; warp 13 issues the MMAs.  Every
// mbarrier wait is bounded; on expiry the kernel records
// DASH_ERR_DEVICE_TIMEOUT and winds down.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace dash {
namespace {

constexpr int kKeys = 128;   // keys per CTA = TMEM lanes
constexpr int kTileRows = 128;
constexpr int kNS = 2;       // Q / dout stages
constexpr int kKeyWarps = 8;           // two per TMEM lane quarter: rows [0, 64) and [64, 128)
constexpr int kInfoWarp0 = kKeyWarps;  // warps 8-11: row data and the summary gradient
constexpr int kProdWarp = 12;
constexpr int kMmaWarpK = 13;
constexpr int kThreadsK = 448;
constexpr int kKeyThreads = kKeyWarps * 32;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
constexpr int kNoLimit = 0x7fffffff;

template <int D, int KB>
struct KLayout {
  static constexpr int KC = D / 64;                 // 128-byte chunks of a row
  static constexpr int kChunk = 128 * 128;          // one chunk of 128 rows
  static constexpr int kTile = KC * kChunk;         // a [128][D] 16-bit tile
  // per stage and row: D, then per block: bias - lse (log2 units, -inf: not
  // attended), the last key position the row sees, dL/dz; then per block the
  // bit mask of the rows with dL/dz != 0
  static constexpr int kInfo = 1 + 3 * KB;
  static constexpr int kInfoBytes = kInfo * kTileRows * 4 + KB * 16;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;                 // [kNS] tiles
  static constexpr int kOffO = kOffQ + kNS * kTile;           // [kNS] tiles
  static constexpr int kOffInfo = kOffO + kNS * kTile;        // [kNS] stage row data
  static constexpr int kOffRed = kOffInfo + kNS * kInfoBytes; // [KB][D] ds, then [KB][D] dk term
  static constexpr int kOffBar = kOffRed + 2 * KB * D * 4;
  static constexpr int kBytes = kOffBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

struct KBars {
  uint64_t kv_full;
  uint64_t qd_full[kNS];     // the stage's Q and dout landed (or: end marker)
  uint64_t desc_ready[kNS];  // the stage's tile index is published
  uint64_t info_full[kNS];   // its row data is written (128 arrivals)
  uint64_t st_empty[kNS];    // MMAs, key threads and row-data threads are done with the stage
  uint64_t s_full;           // S^T and dP^T complete
  uint64_t p_full;           // P^T and dS^T written (256 arrivals)
  uint64_t rd_done;          // the first half of the key threads has read the tile's S^T and dP^T
                             // columns the second half writes over (128 arrivals)
  uint64_t acc_final;        // every MMA complete
  uint32_t tmem_base;
  int abort;
  int tile[kNS];             // the stage's tile, -1 past the last
};

__device__ __forceinline__ void fail(KBars* bars, DeviceStatus* st, int where) {
  raise_status(st, 5 /* DASH_ERR_DEVICE_TIMEOUT */, where);
  atomicExch(&bars->abort, 1);
}

// byte offset of 16-bit element (r, col) of a 128-byte-swizzled [rows][64] chunk
__device__ __forceinline__ int swz16(int r, int col) { return r * 128 + ((((col >> 3) ^ (r & 7))) << 4) + (col & 7) * 2; }

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kThreadsK, 1)
    bwd_key_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      BwdParams p) {
  constexpr int KB = kKeys / BLK;
  using L = KLayout<D, KB>;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescST = tc::idesc_f16(kKeys, kTileRows, kBF16, false, false);
  constexpr uint32_t kIdescKV = tc::idesc_f16(kKeys, D, kBF16, false, true);
  // summary gradient: row-data thread r sums column r % D of the blocks j with
  // j % (128 / D) == r / D (every block when d = 128)
  constexpr int JSTEP = kTileRows / D;
  constexpr int NJ = (KB + JSTEP - 1) / JSTEP;  // blocks per row-data thread

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KBars* bars = reinterpret_cast<KBars*>(smem + L::kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int c0 = grp * KB;  // first block of the CTA
  const int G = p.G;
  const int lgG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  const int P = kTileRows >> lgG;  // positions per tile
  const int n_blocks = (p.S + BLK - 1) / BLK;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  // row data of stage st: dd[128], then per block j: bias - lse, key limit, dL/dz, then the dz masks
  auto info_dd = [&](int st) { return reinterpret_cast<float*>(smem + L::kOffInfo + st * L::kInfoBytes); };
  auto info_bias = [&](int st, int j) { return info_dd(st) + (1 + 3 * j) * kTileRows; };
  auto info_lim = [&](int st, int j) { return reinterpret_cast<int*>(info_dd(st) + (2 + 3 * j) * kTileRows); };
  auto info_dz = [&](int st, int j) { return info_dd(st) + (3 + 3 * j) * kTileRows; };
  auto info_mask = [&](int st, int j) {
    return reinterpret_cast<uint32_t*>(info_dd(st) + L::kInfo * kTileRows) + 4 * j;
  };

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kNS; ++s) {
      tc::mbar_init(&bars->qd_full[s], 1);
      tc::mbar_init(&bars->desc_ready[s], 1);
      tc::mbar_init(&bars->info_full[s], kTileRows);
      tc::mbar_init(&bars->st_empty[s], 1 + kKeyThreads + kTileRows);
    }
    tc::mbar_init(&bars->s_full, 1);
    tc::mbar_init(&bars->p_full, kKeyThreads);
    tc::mbar_init(&bars->rd_done, kKeyThreads / 2);
    tc::mbar_init(&bars->acc_final, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarpK) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) {
    tc::prefetch_tensormap(&tm_q);
    tc::prefetch_tensormap(&tm_do);
    tc::prefetch_tensormap(&tm_k);
    tc::prefetch_tensormap(&tm_v);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kTile);
      for (int kc = 0; kc < L::KC; ++kc) {
        tc::tma_load_4d(smem + L::kOffK + kc * L::kChunk, &tm_k, &bars->kv_full, kc * 64, g, c0 * BLK, b);
        tc::tma_load_4d(smem + L::kOffV + kc * L::kChunk, &tm_v, &bars->kv_full, kc * 64, g, c0 * BLK, b);
      }
    }
    // the tiles whose work list holds one of the CTA's blocks, ascending
    const int t_start = p.causal ? (c0 * BLK) / P : 0;
    const uint32_t sel = (KB == 2 ? 3u : 1u) << (c0 & 31);
    int i = 0;
    bool ok = true;
    for (int t0 = t_start; ok && t0 < p.n_tiles; t0 += 32) {
      const int t = t0 + lane;
      const bool member = t < p.n_tiles && (__ldg(p.tbits + (bg * p.n_tiles + t) * p.n_words + (c0 >> 5)) & sel) != 0u;
      unsigned bal = __ballot_sync(0xffffffffu, member);
      while (bal) {
        const int tile = t0 + __ffs(bal) - 1;
        bal &= bal - 1u;
        if (lane == 0) {
          const int st = i % kNS;
          if (i >= kNS && !tc::mbar_wait(&bars->st_empty[st], ((i / kNS) - 1) & 1)) {
            fail(bars, p.status, 30);
            ok = false;
          } else {
            bars->tile[st] = tile;
            tc::mbar_arrive_expect_tx(&bars->qd_full[st], 2 * L::kTile);
            for (int kc = 0; kc < L::KC; ++kc) {
              tc::tma_load_4d(smem + L::kOffQ + st * L::kTile + kc * L::kChunk, &tm_q, &bars->qd_full[st], kc * 64,
                              g * G, tile * P, b);
              tc::tma_load_4d(smem + L::kOffO + st * L::kTile + kc * L::kChunk, &tm_do, &bars->qd_full[st],
                              kc * 64, g * G, tile * P, b);
            }
            tc::mbar_arrive(&bars->desc_ready[st]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++i;
      }
    }
    if (lane == 0) {
      // the last tile's copies land before the end marker takes a stage
      if (i >= 1) tc::mbar_wait(&bars->qd_full[(i - 1) % kNS], ((i - 1) / kNS) & 1);
      if (ok) {
        const int st = i % kNS;
        if (i >= kNS && !tc::mbar_wait(&bars->st_empty[st], ((i / kNS) - 1) & 1)) {
          fail(bars, p.status, 31);
        } else {
          bars->tile[st] = -1;
          tc::mbar_arrive(&bars->qd_full[st]);
          tc::mbar_arrive(&bars->desc_ready[st]);
        }
      }
      tc::mbar_wait(&bars->kv_full, 0);  // no copy in flight past this point
    }
  } else if (warp == kMmaWarpK) {
    // ------------------------------------------------------------ MMA issuer
    auto wait_all = [&](uint64_t* bar, uint32_t par) { return __all_sync(0xffffffffu, tc::mbar_wait(bar, par)); };
    bool ok = wait_all(&bars->kv_full, 0);
    if (!ok) fail(bars, p.status, 32);
    tc::fence_after_sync();
    const uint64_t kdesc = tc::smem_desc_sw128(smem + L::kOffK, 16, 1024);
    const uint64_t vdesc = tc::smem_desc_sw128(smem + L::kOffV, 16, 1024);
    for (int i = 0; ok; ++i) {
      const int st = i % kNS;
      if (!wait_all(&bars->qd_full[st], (i / kNS) & 1)) {
        fail(bars, p.status, 33);
        break;
      }
      if (bars->tile[st] < 0) break;
      tc::fence_after_sync();
      const uint64_t qdesc = tc::smem_desc_sw128(smem + L::kOffQ + st * L::kTile, 16, 1024);
      const uint64_t odesc = tc::smem_desc_sw128(smem + L::kOffO + st * L::kTile, 16, 1024);
      // S^T = K Q^T and dP^T = V dout^T: contraction over d, 16 at a time
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t off = (uint64_t)((((k >> 2) * L::kChunk) + (k & 3) * 32) >> 4);
        tc::mma_f16_ss_w(tmem + kColS, kdesc + off, qdesc + off, kIdescST, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t off = (uint64_t)((((k >> 2) * L::kChunk) + (k & 3) * 32) >> 4);
        tc::mma_f16_ss_w(tmem + kColDP, vdesc + off, odesc + off, kIdescST, k > 0 ? 1u : 0u);
      }
      tc::mma_commit_w(&bars->s_full);
      if (!wait_all(&bars->p_full, i & 1)) {
        fail(bars, p.status, 34);
        break;
      }
      tc::fence_after_sync();
      // dV += P^T dout and dK += dS^T Q: contraction over the tile's 128 rows,
      // B (dout, Q) MN-major: 16 rows per MMA, 64-column chunks kChunk apart
      const uint64_t odesc_mn = tc::smem_desc_sw128(smem + L::kOffO + st * L::kTile, L::kChunk, 1024);
      const uint64_t qdesc_mn = tc::smem_desc_sw128(smem + L::kOffQ + st * L::kTile, L::kChunk, 1024);
#pragma unroll
      for (int k = 0; k < kTileRows / 16; ++k)
        tc::mma_f16_ts_w(tmem + kColDV, tmem + kColS + k * 8, odesc_mn + (uint64_t)((k * 2048) >> 4), kIdescKV,
                         (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < kTileRows / 16; ++k)
        tc::mma_f16_ts_w(tmem + kColDK, tmem + kColDP + k * 8, qdesc_mn + (uint64_t)((k * 2048) >> 4), kIdescKV,
                         (i > 0 || k > 0) ? 1u : 0u);
      tc::mma_commit_w(&bars->st_empty[st]);
    }
    // acc_final completes once every MMA issued above has
    tc::mma_commit_w(&bars->acc_final);
    tc::mbar_wait(&bars->acc_final, 0);
  } else if (warp >= kInfoWarp0) {
    // ------------------------------------------------------------ row data and the summary gradient
    const int r = threadIdx.x - kInfoWarp0 * 32;  // tile row (first role); column and blocks (second)
    const int col = r % D, j0 = r / D;
    float dsacc[NJ];
#pragma unroll
    for (int m = 0; m < NJ; ++m) dsacc[m] = 0.f;
    for (int i = 0;; ++i) {
      const int st = i % kNS;
      if (!tc::mbar_wait(&bars->desc_ready[st], (i / kNS) & 1)) {
        fail(bars, p.status, 35);
        break;
      }
      const int tile = bars->tile[st];
      if (tile >= 0) {
        const int pos = tile * P + (r >> lgG);
        const int hh = r & (G - 1), h = g * G + hh;
        const bool valid = pos < p.S;
        const int64_t hrow = ((int64_t)b * p.H + h) * p.S + pos;
        const float lse = valid ? __ldg(p.lse + hrow) : 0.f;
        info_dd(st)[r] = valid ? __ldg(p.dd + hrow) : 0.f;
        const int t = pos / BLK;
        const int n_cand = p.causal ? t : n_blocks - 1;
        const int64_t row = bg * p.S + pos;
        const uint32_t* rm = p.rmask + row * p.n_words;
        const int32_t* rk = p.rrank + row * p.n_words;
#pragma unroll
        for (int j = 0; j < KB; ++j) {
          const int c = c0 + j;
          float bias = kNegInf, dz = 0.f;
          int lim = kNoLimit;
          if (valid && c < n_blocks) {
            if (c == t) {
              bias = n_cand > 0 ? p.sigma * logf(1.0f / (float)n_cand) * kLog2e : 0.f;
              if (p.causal) lim = pos;
            } else if (!p.causal || c < t) {
              const uint32_t word = __ldg(rm + (c >> 5));
              const int before = __ldg(rk + (c >> 5));  // selections in the words below
              if ((word >> (c & 31)) & 1u) {
                const int e = before + __popc(word & ((1u << (c & 31)) - 1u));
                bias = p.sigma * __ldg(p.logp + row * p.t_cap + e) * kLog2e;
                dz = __ldg(p.dz + (row * p.t_cap + e) * G + hh);
              }
            }
          }
          info_bias(st, j)[r] = bias == kNegInf ? kNegInf : bias - lse;
          info_lim(st, j)[r] = lim;
          info_dz(st, j)[r] = dz;
          const unsigned m = __ballot_sync(0xffffffffu, dz != 0.f);
          if (lane == 0) info_mask(st, j)[warp - kInfoWarp0] = m;
        }
      }
      tc::mbar_arrive(&bars->info_full[st]);
      if (tile < 0) break;
      // summary gradient: sum over the rows with dL/dz != 0 of dL/dz(row, block) q_row,
      // rows in ascending order (deterministic); needs every warp's dz masks and this stage's Q
      if (!tc::mbar_wait(&bars->info_full[st], (i / kNS) & 1) || !tc::mbar_wait(&bars->qd_full[st], (i / kNS) & 1)) {
        fail(bars, p.status, 39);
        break;
      }
      // one pass over the tile's rows: each Q value is loaded once for the
      // thread's blocks (rows with dL/dz = 0 add zero)
      bool any = false;
#pragma unroll
      for (int m = 0; m < NJ; ++m) {
        const int j = j0 + m * JSTEP;
        if (j < KB) {
          const uint32_t* mk = info_mask(st, j);
          any = any || (mk[0] | mk[1] | mk[2] | mk[3]) != 0u;
        }
      }
      if (any) {
        const uint8_t* qc = smem + L::kOffQ + st * L::kTile + (col >> 6) * L::kChunk;
        float acc[NJ][2];
#pragma unroll
        for (int m = 0; m < NJ; ++m) acc[m][0] = acc[m][1] = 0.f;
#pragma unroll 4
        for (int rr = 0; rr < kTileRows; rr += 2) {
          const float q0 = Elt<T>::load1(reinterpret_cast<const T*>(qc + swz16(rr, col & 63)));
          const float q1 = Elt<T>::load1(reinterpret_cast<const T*>(qc + swz16(rr + 1, col & 63)));
#pragma unroll
          for (int m = 0; m < NJ; ++m) {
            const int j = j0 + m * JSTEP;
            if (j < KB) {
              const float2 z = *reinterpret_cast<const float2*>(info_dz(st, j) + rr);
              acc[m][0] = fmaf(z.x, q0, acc[m][0]);
              acc[m][1] = fmaf(z.y, q1, acc[m][1]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < NJ; ++m) dsacc[m] += acc[m][0] + acc[m][1];
      }
      tc::mbar_arrive(&bars->st_empty[st]);
    }

    // ---- epilogue part 1: summary gradient, block means and the stage-0 term of dk
    float* red = reinterpret_cast<float*>(smem + L::kOffRed);  // [KB][D] ds, then [KB][D] dk term
    const float gam = rsqrtf((float)D);
    const bool kv_ok = tc::mbar_wait(&bars->kv_full, 0);
#pragma unroll
    for (int m = 0; m < NJ; ++m) {
      const int j = j0 + m * JSTEP;
      if (j < KB) {
        const int cj = c0 + j;
        const int nk = max(1, min(BLK, p.S - cj * BLK));
        float kb = 0.f;
        if (kv_ok)
          for (int kk = 0; kk < nk; ++kk)
            kb += Elt<T>::load1(reinterpret_cast<const T*>(smem + L::kOffK + (col >> 6) * L::kChunk +
                                                            swz16(j * BLK + kk, col & 63)));
        const float dsv = gam * dsacc[m];
        red[j * D + col] = dsv;
        if (cj < n_blocks) {
          p.kbar[(bg * p.t_cap + cj) * D + col] = kb / (float)nk;
          p.ds[(bg * p.t_cap + cj) * D + col] = dsv;
        }
      }
    }
    asm volatile("bar.sync 2, 128;\n" ::: "memory");
#pragma unroll
    for (int m = 0; m < NJ; ++m) {
      const int j = j0 + m * JSTEP;
      if (j < KB) {
        const int nk = max(1, min(BLK, p.S - (c0 + j) * BLK));
        const float* wr = p.w_s + (int64_t)col * D;
        float a = 0.f;
        for (int jj = 0; jj < D; ++jj) a = fmaf(__ldg(wr + jj), red[j * D + jj], a);
        red[KB * D + j * D + col] = a / (float)nk;
      }
    }
    // hand the dk term to the key threads
    asm volatile("bar.sync 3, %0;\n" ::"n"(kKeyThreads + kTileRows) : "memory");
  } else {
    // ------------------------------------------------------------ key threads (warps 0-7)
    const int q4 = warp & 3, half = warp >> 2;
    const int k = q4 * 32 + lane;  // key of the CTA = TMEM lane
    const int blk = k / BLK;
    const int key_pos = c0 * BLK + k;
    const bool kvalid = key_pos < p.S;
    const uint32_t tb = tmem + ((uint32_t)(q4 * 32) << 16);
    const float sc = rsqrtf((float)D) * kLog2e;
    bool ok = true;
    int n_done = 0;  // tiles processed (0: dV and dK were never written in TMEM)
    for (int i = 0;; ++i) {
      const int st = i % kNS;
      if (!tc::mbar_wait(&bars->info_full[st], (i / kNS) & 1)) {
        fail(bars, p.status, 36);
        ok = false;
        break;
      }
      const int tile = bars->tile[st];
      if (tile < 0) break;
      if (!tc::mbar_wait(&bars->s_full, i & 1)) {
        fail(bars, p.status, 37);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const float* dd = info_dd(st);
      const float* bias = info_bias(st, blk);
      const int* lim = info_lim(st, blk);
      // P^T and dS^T go back packed two rows per column over the first halves
      // of the S^T and dP^T columns: the second half's writes land on columns
      // the first half reads, so they wait for those reads
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int ch = half * 2 + cc;  // 32-row chunk of this thread's half
        uint32_t sv[32], pv[32];
        tc::tmem_ld32(tb + kColS + ch * 32, sv);
        tc::tmem_ld32(tb + kColDP + ch * 32, pv);
        tc::tmem_wait_ld();
        if (half == 0 && cc == 1) {
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->rd_done);
        }
        uint32_t pw[16], dw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int r0 = ch * 32 + e;
          const float4 bi = *reinterpret_cast<const float4*>(bias + r0);
          const int4 li = *reinterpret_cast<const int4*>(lim + r0);
          const float4 dv4 = *reinterpret_cast<const float4*>(dd + r0);
          const float bis[4] = {bi.x, bi.y, bi.z, bi.w};
          const int lis[4] = {li.x, li.y, li.z, li.w};
          const float dvs[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
          float pr[4], ds[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool on = kvalid && bis[u] != kNegInf && key_pos <= lis[u];
            pr[u] = on ? tc::ex2(fmaf(__uint_as_float(sv[e + u]), sc, bis[u])) : 0.f;
            ds[u] = pr[u] * (__uint_as_float(pv[e + u]) - dvs[u]);
          }
          pw[e >> 1] = pack2<T>(pr[0], pr[1]);
          pw[(e >> 1) + 1] = pack2<T>(pr[2], pr[3]);
          dw[e >> 1] = pack2<T>(ds[0], ds[1]);
          dw[(e >> 1) + 1] = pack2<T>(ds[2], ds[3]);
        }
        if (half == 1 && cc == 0) {
          if (!tc::mbar_wait(&bars->rd_done, i & 1)) {
            fail(bars, p.status, 40);
            ok = false;
          }
          tc::fence_after_sync();
        }
        tc::tmem_st16(tb + kColS + ch * 16, pw);
        tc::tmem_st16(tb + kColDP + ch * 16, dw);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full);
      tc::mbar_arrive(&bars->st_empty[st]);
      ++n_done;
    }

    // ---- epilogue part 2: dk and dv (each thread half of its key's columns)
    const bool done = tc::mbar_wait(&bars->acc_final, 0);
    tc::fence_after_sync();
    asm volatile("bar.sync 3, %0;\n" ::"n"(kKeyThreads + kTileRows) : "memory");  // the dk term is ready
    const float* red = reinterpret_cast<const float*>(smem + L::kOffRed);
    if (done) {
      const float ksc = rsqrtf((float)D);
      const float* dkb = red + KB * D + blk * D;
      float* dkg = static_cast<float*>(const_cast<void*>(p.dk.data)) + (int64_t)b * p.dk.sb +
                   (int64_t)(kvalid ? key_pos : 0) * p.dk.ss + (int64_t)g * p.dk.sh;
      float* dvg = static_cast<float*>(const_cast<void*>(p.dv.data)) + (int64_t)b * p.dv.sb +
                   (int64_t)(kvalid ? key_pos : 0) * p.dv.ss + (int64_t)g * p.dv.sh;
#pragma unroll 1
      for (int cc = half * (D / 64); cc < (half + 1) * (D / 64); ++cc) {
        uint32_t v[32], w[32];
        tc::tmem_ld32(tb + kColDV + cc * 32, v);
        tc::tmem_ld32(tb + kColDK + cc * 32, w);
        tc::tmem_wait_ld();
        if (n_done == 0) {
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = w[q] = 0u;
        }
        if (kvalid) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int col = cc * 32 + q * 4;
            *reinterpret_cast<float4*>(dvg + col) =
                make_float4(__uint_as_float(v[q * 4]), __uint_as_float(v[q * 4 + 1]), __uint_as_float(v[q * 4 + 2]),
                            __uint_as_float(v[q * 4 + 3]));
            *reinterpret_cast<float4*>(dkg + col) = make_float4(
                fmaf(__uint_as_float(w[q * 4]), ksc, dkb[col]), fmaf(__uint_as_float(w[q * 4 + 1]), ksc, dkb[col + 1]),
                fmaf(__uint_as_float(w[q * 4 + 2]), ksc, dkb[col + 2]),
                fmaf(__uint_as_float(w[q * 4 + 3]), ksc, dkb[col + 3]));
          }
        }
      }
    } else if (ok) {
      fail(bars, p.status, 38);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarpK) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Bit masks of the stage-2 tiles' work lists: bit c of tile t set iff block c
// is in the list (one warp per tile).
__global__ void __launch_bounds__(256) tile_bits_kernel(const int32_t* ulist, const int32_t* ucnt, int64_t n_lists,
                                                        int64_t t_cap, uint32_t* bits, int n_words) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  if (t >= n_lists) return;
  uint32_t* out = bits + t * n_words;
  for (int w = lane; w < n_words; w += 32) out[w] = 0u;
  __syncwarp();
  const int n = min(max(ucnt[t], 0), (int)t_cap);
  for (int e = lane; e < n; e += 32) {
    const int c = ulist[t * t_cap + e];
    if (c >= 0 && c < n_words * 32) atomicOr(out + (c >> 5), 1u << (c & 31));
  }
}

template <typename T, int D, int BLK>
cudaError_t launch_key_tc(const BwdParams& p, cudaStream_t stream) {
  constexpr int KB = kKeys / BLK;
  using L = KLayout<D, KB>;
  CUtensorMap mq, mdo, mk, mv;
  const int P = kTileRows / p.G;
  if (!make_map(&mq, p.q, p.dtype, p.B, p.S, p.H, D, p.G, P) ||
      !make_map(&mdo, p.dout, p.dtype, p.B, p.S, p.H, D, p.G, P) ||
      !make_map(&mk, p.k, p.dtype, p.B, p.S, p.Hkv, D, 1, kKeys) ||
      !make_map(&mv, p.v, p.dtype, p.B, p.S, p.Hkv, D, 1, kKeys))
    return cudaErrorInvalidValue;
  auto kern = bwd_key_tc_kernel<T, D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const int n_groups = (int)((p.t_cap + KB - 1) / KB);
  kern<<<dim3(n_groups, p.Hkv, p.B), kThreadsK, L::kAlloc, stream>>>(mq, mdo, mk, mv, p);
  return cudaGetLastError();
}

// Exclusive prefix of each row's selection counts over its mask words:
// rank[row][w] = number of selected blocks below block 32 w (one warp per row).
__global__ void __launch_bounds__(256) rank_kernel(const uint32_t* mask, int64_t rows, int n_words, int32_t* rank) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const uint32_t* m = mask + row * n_words;
  int32_t* out = rank + row * n_words;
  int base = 0;
  for (int w0 = 0; w0 < n_words; w0 += 32) {
    const int n = w0 + lane < n_words ? __popc(m[w0 + lane]) : 0;
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (w0 + lane < n_words) out[w0 + lane] = base + incl - n;
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
}

}  // namespace

cudaError_t launch_row_ranks(const uint32_t* mask, int64_t rows, int n_words, int32_t* rank, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  rank_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(mask, rows, n_words, rank);
  return cudaGetLastError();
}

cudaError_t launch_tile_bits(const int32_t* ulist, const int32_t* ucnt, int64_t n_lists, int64_t t_cap, uint32_t* bits,
                             int n_words, cudaStream_t stream) {
  if (n_lists <= 0) return cudaSuccess;
  tile_bits_kernel<<<(unsigned)((n_lists + 7) / 8), 256, 0, stream>>>(ulist, ucnt, n_lists, t_cap, bits, n_words);
  return cudaGetLastError();
}

cudaError_t launch_bwd_key_tc(const BwdParams& p, cudaStream_t stream) {
  if (p.dtype == 1) {
    if (p.D == 128) return p.block == 128 ? launch_key_tc<__half, 128, 128>(p, stream) : launch_key_tc<__half, 128, 64>(p, stream);
    return p.block == 128 ? launch_key_tc<__half, 64, 128>(p, stream) : launch_key_tc<__half, 64, 64>(p, stream);
  }
  if (p.D == 128)
    return p.block == 128 ? launch_key_tc<__nv_bfloat16, 128, 128>(p, stream)
                          : launch_key_tc<__nv_bfloat16, 128, 64>(p, stream);
  return p.block == 128 ? launch_key_tc<__nv_bfloat16, 64, 128>(p, stream)
                        : launch_key_tc<__nv_bfloat16, 64, 64>(p, stream);
}

}  // namespace dash
