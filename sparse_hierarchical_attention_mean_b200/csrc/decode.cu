// Decode step: stage 1 against cached summaries and the split-KV stage 2.
//
// "Stage 0: local chunk summary" (a chunk's summary is cached once the chunk
// is complete, so decoding never recomputes it), "Stage 1: entmax chunk
// routing" and "Stage 2: prior-induced sparse softmax" of the DashAttention
// technical summary, for one new query token per sequence; the pages report
// decoding speed "in the memory-bound regime", which is what these kernels
// are shaped for: every byte of the cached summaries and of the selected
// K/V blocks is read once.
//
//  score_decode      (b, g, 64-block chunk) CTAs; a warp reads 8 summary
//                    rows (coalesced fp32) and dots them with the G query
//                    heads; a warp reduce-scatter finishes the G*8 sums.
//  entmax_decode     one CTA per (b, g): tau per head (warp per head), GQA
//                    mean, ballot/popc compaction, and the split-KV work
//                    items (chunks of selected blocks) appended with one
//                    atomic per (b, g).
//  attend_decode_mma persistent CTAs over the work items: K/V rows of the
//                    selected blocks (dense or paged cache) stream through a
//                    cp.async ring; each warp owns 16 tokens of a 64-token
//                    step, takes both products on the tensor cores with
//                    warp-level MMAs, keeps an online softmax per head; the
//                    4 warps merge into one (m, l, o) partial per item.
//  combine_decode    log-sum-exp merge of the partials of each (b, g).
//  attend_shard, cp_merge  context parallelism: stage 2 over one rank's
//                    tokens into per-head partials (CUDA cores, no
//                    workspace), and their merge.
//  shard_items, combine_partial  context parallelism on the split-KV path:
//                    the shard's range of each list cut into work items for
//                    attend_decode_mma, and its per-head partials.
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"

namespace dash {
namespace {

__device__ __forceinline__ int clamp_len(const int32_t* seqlens, int b, int lmax, DeviceStatus* st) {
  int L = seqlens[b];
  if (L < 1 || L > lmax) {
    raise_status(st, 1 /* DASH_ERR_INVALID_ARGUMENT */, 100 + b);
    L = L < 1 ? 1 : lmax;
  }
  return L;
}

// ------------------------------------------------------------------ scores
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) score_decode_kernel(DecodeParams p) {
  constexpr int DL = D / 32;
  constexpr int NV = 8 * G;
  const int b = blockIdx.z, g = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = clamp_len(p.seqlens, b, p.Lmax, p.status);
  const int N = min((L - 1) / p.block, p.c_hi);  // scored here: candidates c_lo <= c < N
  const int c0 = blockIdx.x * 64 + warp * 8;
  if (c0 >= N || c0 + 8 <= p.c_lo) return;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  float qv[G][DL];
  const T* q = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL; ++e) qv[h][e] = Elt<T>::load1(q + (int64_t)(g * G + h) * p.q.sh + lane * DL + e);
  float v[NV];
  const float* sb = p.summaries + bg * p.summ_cap * D + lane * DL;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float s[DL];
    if (c0 + i < N && c0 + i >= p.c_lo) {
      const int64_t si = c0 + i - p.c_lo;
      if constexpr (DL == 4) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(sb + si * D));
        s[0] = x.x, s[1] = x.y, s[2] = x.z, s[3] = x.w;
      } else {
        const float2 x = __ldg(reinterpret_cast<const float2*>(sb + si * D));
        s[0] = x.x, s[1] = x.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < DL; ++e) s[e] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) a = fmaf(qv[h][e], s[e], a);
      v[i * G + h] = a;
    }
  }
  warp_transpose_reduce<NV>(v, lane);
  const float coef = (p.alpha - 1.0f) * rsqrtf((float)D);
  if constexpr (NV >= 32) {
#pragma unroll
    for (int j = 0; j < NV / 32; ++j) {
      const int i = lane * (NV / 32) + j;
      const int c = c0 + i / G, h = i % G;
      if (c < N && c >= p.c_lo) p.scores[(bg * G + h) * p.t_cap + c] = coef * v[j];
    }
  } else {
    constexpr int SH = NV == 16 ? 1 : (NV == 8 ? 2 : 0);
    if ((lane & ((1 << SH) - 1)) == 0) {
      const int i = lane >> SH;
      const int c = c0 + i / G, h = i % G;
      if (c < N && c >= p.c_lo) p.scores[(bg * G + h) * p.t_cap + c] = coef * v[0];
    }
  }
}

// ------------------------------------------------------------------ entmax + compaction
__global__ void __launch_bounds__(256) entmax_decode_kernel(DecodeParams p) {
  extern __shared__ __align__(16) float xs[];  // [G][t_cap]
  __shared__ float tau_s[8];
  const int b = blockIdx.y, g = blockIdx.x;
  const int G = p.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = clamp_len(p.seqlens, b, p.Lmax, nullptr);
  const int N = (L - 1) / p.block;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const float pw = 1.0f / (p.alpha - 1.0f);
  const int kind = entmax_kind(p.alpha);
  for (int i = threadIdx.x; i < G * N; i += blockDim.x) {
    const int h = i / N, c = i % N;
    xs[h * p.t_cap + c] = p.scores[(bg * G + h) * p.t_cap + c];
  }
  __syncthreads();
  for (int h = warp; h < G; h += blockDim.x / 32) {
    const float tau = N > 0 ? warp_entmax_tau(xs + h * p.t_cap, N, p.alpha, lane) : 0.f;
    if (lane == 0) tau_s[h] = tau;
  }
  __syncthreads();
  if (warp == 0) {
    int32_t* idx = p.idx + bg * p.t_cap;
    float* logp = p.logp + bg * p.t_cap;
    int off = 0;
    for (int c0 = 0; c0 < N; c0 += 32) {
      const int c = c0 + lane;
      float pb = 0.f;
      if (c < N) {
        for (int h = 0; h < G; ++h) {
          const float u = xs[h * p.t_cap + c] - tau_s[h];
          if (u > 0.f) pb += pow_pw(u, pw, kind);
        }
        pb /= (float)G;
      }
      const bool sel = pb > 0.f;
      const unsigned m = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int o = off + __popc(m & ((1u << lane) - 1u));
        idx[o] = c;
        logp[o] = logf(pb);
      }
      off += __popc(m);
    }
    if (lane == 0) {
      p.cnt[bg] = off;
      if (p.items) {
        const int n_it = (off + 1 + p.chunk_blocks - 1) / p.chunk_blocks;
        const int base = atomicAdd(p.n_items, n_it);
        p.pair_base[bg] = base;
        for (int k = 0; k < n_it; ++k) {
          p.items[2 * (base + k)] = (int32_t)bg;
          p.items[2 * (base + k) + 1] = k;
        }
      }
    }
  }
  if (p.tau || p.p_dense) {
    for (int h = warp; h < G; h += blockDim.x / 32) {
      const int64_t hrow = (int64_t)b * p.H + g * G + h;
      if (p.tau && lane == 0) p.tau[hrow] = tau_s[h];
      if (p.p_dense) {
        for (int c = lane; c < p.t_cap; c += 32) {
          float v = 0.f;
          if (c < N) {
            const float u = xs[h * p.t_cap + c] - tau_s[h];
            if (u > 0.f) v = pow_pw(u, pw, kind);
          }
          p.p_dense[hrow * p.t_cap + c] = v;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ split-KV attention
constexpr int kStep = 64;  // tokens per pipeline step
constexpr int kWarps = 4;  // 16 tokens per warp per step

// Split-KV attention over the work items (chunks of selected blocks of one
// (sequence, KV head)), one partial per item.  The two per-warp products run
// on the tensor cores through warp-level mma (m16n8k16, fp32 accumulate): a KV head has only G <= 8 query rows, far below the
// 64-row minimum of the 5th-generation MMA, and the kernel is HBM-bound, so
// the MMAs only serve to take the dot products off the issue slots.
//   S^T (16 x 8 tokens) = Qpad (16 x D) K^T: rows are the G heads (zero
//   padding above G), B fragments come from the K rows by ldmatrix;
//   O (16 x D) += P (16 x 16 tokens) V: P is the S accumulator re-packed in
//   registers (the accumulator layout of two 8-token tiles is the A layout of
//   one 16-token tile), V fragments by ldmatrix.trans.
// K/V stream through a kDStages-deep cp.async ring; each row of 16-byte
// chunks is stored XOR-swizzled by (token & 7) so the ldmatrix row reads are
// free of bank conflicts.  Each warp owns 16 tokens of every 64-token step and
// keeps its own online softmax; O is rescaled only when a head's reference
// max grows by more than 2^8 (P <= 256, exact after the final division).
constexpr int kDStages = 3;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kWarps * 32) attend_decode_mma_kernel(DecodeParams p) {
  static_assert(G <= 8, "heads of a group must fit the 8 live MMA rows");
  constexpr int NCH = D / 8;       // 16-byte chunks per row
  constexpr int NT = D / 8;        // 8-wide d tiles of O
  constexpr int KS = D / 16;       // k steps of S
  constexpr int kStageElems = kStep * D;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  T* Ks = reinterpret_cast<T*>(smem_raw);               // [kDStages][kStep][D] swizzled
  T* Vs = Ks + kDStages * kStageElems;                  // [kDStages][kStep][D] swizzled
  float* mbuf = reinterpret_cast<float*>(Vs + kDStages * kStageElems);  // [kWarps][G]
  float* lbuf = mbuf + kWarps * G;                      // [kWarps][G]
  float* obuf = lbuf + kWarps * G;                      // [kWarps][G][D]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row group / thread in group
  const int n_items = *p.n_items;
  const float qk_scale = rsqrtf((float)D) * kLog2e;
  const uint32_t ks_base = smem_u32(Ks), vs_base = smem_u32(Vs);

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int bg = p.items[2 * item], chunk = p.items[2 * item + 1];
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int L = clamp_len(p.seqlens, b, p.Lmax, nullptr);
    const int pos = L - 1;
    const int t = pos / p.block;
    const int N = t;
    // list entries [e_lo, e_hi) and, when held, the diagonal block (entry e_hi)
    int e_lo = 0, e_hi = p.cnt[bg];
    bool diag_held = true;
    if (p.shard) {
      e_lo = p.shard[4 * bg];
      e_hi = p.shard[4 * bg + 1];
      diag_held = p.shard[4 * bg + 2] != 0;
    }
    const int e_begin = e_lo + chunk * p.chunk_blocks;
    const int e_end = min(e_begin + p.chunk_blocks, diag_held ? e_hi + 1 : e_hi);
    const bool has_diag = diag_held && e_end == e_hi + 1;
    const int spb = p.block / kStep;
    const int n_diag = has_diag ? (pos - t * p.block) / kStep + 1 : 0;
    const int n_sel = (has_diag ? e_end - 1 : e_end) - e_begin;
    const int n_sub = n_sel * spb + n_diag;
    const int32_t* idx = p.idx + (int64_t)bg * p.t_cap;
    const float* logp = p.logp + (int64_t)bg * p.t_cap;
    const float beta = N > 0 ? p.sigma * logf(1.0f / (float)N) : 0.0f;
    const T* kg = static_cast<const T*>(p.k.data) + (int64_t)g * p.k.sh;
    const T* vg = static_cast<const T*>(p.v.data) + (int64_t)g * p.v.sh;

    auto sub_tok0 = [&](int s) -> int {
      if (s < n_sel * spb) return idx[e_begin + s / spb] * p.block + (s % spb) * kStep;
      return t * p.block + (s - n_sel * spb) * kStep;
    };
    auto load = [&](int s) {
      if (s < n_sub) {
        int tok0 = sub_tok0(s);
        // a shard reads only its own rows (ascending lists keep every step
        // inside it; anything else is zero-filled)
        const bool in_shard = !p.shard || (tok0 >= p.tok_lo && tok0 + kStep <= p.tok_lo + p.tok_n);
        // first row of the step: a step never crosses a block, so a paged
        // cache needs one page lookup per step
        int64_t kr0, vr0;
        if (p.block_table) {
          const int64_t page = p.block_table[(int64_t)b * p.max_blocks + tok0 / p.block];
          kr0 = page * p.k.sb + (int64_t)(tok0 % p.block) * p.k.ss;
          vr0 = page * p.v.sb + (int64_t)(tok0 % p.block) * p.v.ss;
        } else {
          const int row0 = in_shard ? tok0 - p.tok_lo : 0;
          kr0 = (int64_t)b * p.k.sb + (int64_t)row0 * p.k.ss;
          vr0 = (int64_t)b * p.v.sb + (int64_t)row0 * p.v.ss;
        }
        T* kd = Ks + (s % kDStages) * kStageElems;
        T* vd = Vs + (s % kDStages) * kStageElems;
        for (int i = tid; i < kStep * NCH; i += kWarps * 32) {
          const int r = i / NCH, c = i % NCH;
          const bool ok = in_shard && tok0 + r < L;  // rows past the context are zero-filled
          const int pc = c ^ (r & 7);
          const int rr = ok ? r : 0;
          cp_async16(kd + r * D + pc * 8, kg + kr0 + (int64_t)rr * p.k.ss + c * 8, ok);
          cp_async16(vd + r * D + pc * 8, vg + vr0 + (int64_t)rr * p.v.ss + c * 8, ok);
        }
      }
      cp_async_commit();
    };

    // query A fragments: rows = heads (row gq < G), 16 d per k step
    uint32_t qa[KS][2];
    {
      const T* q = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)(g * G + (gq < G ? gq : 0)) * p.q.sh;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = gq < G ? *reinterpret_cast<const uint32_t*>(q + kk * 16 + 2 * tq) : 0u;
        qa[kk][1] = gq < G ? *reinterpret_cast<const uint32_t*>(q + kk * 16 + 8 + 2 * tq) : 0u;
      }
    }
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_used = kNegInf, lpart = 0.f;

#pragma unroll
    for (int s = 0; s < kDStages - 1; ++s) load(s);
    for (int s = 0; s < n_sub; ++s) {
      load(s + kDStages - 1);
      cp_async_wait<kDStages - 1>();
      __syncthreads();
      const int st = s % kDStages;
      const uint32_t kst = ks_base + (uint32_t)(st * kStageElems * sizeof(T));
      const uint32_t vst = vs_base + (uint32_t)(st * kStageElems * sizeof(T));
      const bool diag = s >= n_sel * spb;
      const float bias = (diag ? beta : p.sigma * logp[e_begin + s / spb]) * kLog2e;
      const int tok0 = sub_tok0(s) + warp * 16;

      // S^T = Q K^T for this warp's 16 tokens (two 8-token tiles)
      float sacc[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
      {
        const int m = lane >> 3, rr = lane & 7;
        const int tok = warp * 16 + (m >> 1) * 8 + rr;  // row within the stage
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const int c = 2 * kk + (m & 1);
          uint32_t bf[4];
          ldsm_x4(kst + (uint32_t)((tok * D + ((c ^ (tok & 7)) * 8)) * sizeof(T)), bf);
          const uint32_t a[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
          mma16816<T>(sacc[0], a, bf[0], bf[1]);
          mma16816<T>(sacc[1], a, bf[2], bf[3]);
        }
      }
      // logits (log2 domain) of head gq for tokens 2tq, 2tq+1, 8+2tq, 9+2tq
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tk = tok0 + (e >> 1) * 8 + 2 * tq + (e & 1);
        x[e] = tk <= pos ? fmaf(sacc[e >> 1][e & 1], qk_scale, bias) : kNegInf;
      }
      float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float corr = 1.0f;
      bool resc = false;
      if (mx != kNegInf) {
        if (m_used == kNegInf) {
          m_used = mx;
        } else if (mx > m_used + 8.0f) {
          corr = exp2f(m_used - mx);
          m_used = mx;
          resc = true;
        }
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= corr;
          o[n][1] *= corr;
        }
        lpart *= corr;
      }
      float pe[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pe[e] = m_used == kNegInf ? 0.f : exp2f(x[e] - m_used);
      lpart += (pe[0] + pe[1]) + (pe[2] + pe[3]);
      const uint32_t pa[4] = {pack2<T>(pe[0], pe[1]), 0u, pack2<T>(pe[2], pe[3]), 0u};

      // O += P V: B fragments of two 8-wide d tiles per ldmatrix
      {
        const int m = lane >> 3, rr = lane & 7;
        const int tok = warp * 16 + (m & 1) * 8 + rr;
#pragma unroll
        for (int j = 0; j < NT / 2; ++j) {
          const int c = 2 * j + (m >> 1);
          uint32_t bf[4];
          ldsm_x4_t(vst + (uint32_t)((tok * D + ((c ^ (tok & 7)) * 8)) * sizeof(T)), bf);
          mma16816<T>(o[2 * j], pa, bf[0], bf[1]);
          mma16816<T>(o[2 * j + 1], pa, bf[2], bf[3]);
        }
      }
      __syncthreads();  // the stage is free for the load issued next iteration
    }
    cp_async_wait<0>();

    // merge the 4 warps: rows gq < G hold head gq; lanes of a row group split d
    float l = lpart;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (gq < G) {
      if (tq == 0) {
        mbuf[warp * G + gq] = m_used;
        lbuf[warp * G + gq] = l;
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        obuf[(warp * G + gq) * D + n * 8 + 2 * tq] = o[n][0];
        obuf[(warp * G + gq) * D + n * 8 + 2 * tq + 1] = o[n][1];
      }
    }
    __syncthreads();
    const int64_t slot = (int64_t)p.pair_base[bg] + chunk;
    for (int i = tid; i < G * D; i += kWarps * 32) {
      const int h = i / D, e = i % D;
      float M = kNegInf;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mbuf[w * G + h]);
      const float Mu = M == kNegInf ? 0.f : M;
      float acc = 0.f, lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(mbuf[w * G + h] - Mu);
        acc += f * obuf[(w * G + h) * D + e];
        lsum += f * lbuf[w * G + h];
      }
      p.part_o[(slot * G + h) * D + e] = acc;
      if (e == 0) {
        p.part_ml[(slot * G + h) * 2] = M;
        p.part_ml[(slot * G + h) * 2 + 1] = lsum;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ context-parallel shard attention
// One CTA per (KV head, sequence) over this shard's part of the selected
// blocks (a contiguous range of the ascending list) and, when the shard
// holds it, the diagonal block; 16-token units go round-robin to the 4
// warps, each keeping an online softmax per head (logits by a warp
// reduce-scatter, P broadcast through shared memory).  The 4 warps merge into
// one partial per head: o relative to the reference max m (log2 units) and l.
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) attend_shard_kernel(DecodeParams p) {
  constexpr int DL = D / 32;
  constexpr int NV = 16 * G;
  constexpr int NVL = NV >= 32 ? NV / 32 : 1;
  constexpr int GH = G >= 2 ? G / 2 : 1;
  constexpr int W = 4;
  __shared__ float pbuf[W][16 * G];
  __shared__ float mbuf[W][G], lbuf[W][G];
  __shared__ float obuf[W][G][D];
  __shared__ int erange[2];
  const int g = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int L = clamp_len(p.seqlens, b, p.Lmax, nullptr);
  const int pos = L - 1, t = pos / p.block, N = t;
  const float beta = N > 0 ? p.sigma * logf(1.0f / (float)N) : 0.0f;
  const int c_lo = p.tok_lo / p.block, c_hi = (p.tok_lo + p.tok_n) / p.block;
  const int cnt = min(max(p.cnt[bg], 0), (int)p.t_cap);
  const int32_t* idx = p.idx + bg * p.t_cap;
  const float* logp = p.logp + bg * p.t_cap;
  if (warp == 0) {
    int nlo = 0, nhi = 0;
    for (int e = lane; e < cnt; e += 32) {
      const int c = idx[e];
      nlo += c < c_lo ? 1 : 0;
      nhi += c < c_hi ? 1 : 0;
    }
    nlo = warp_sum_i(nlo);
    nhi = warp_sum_i(nhi);
    if (lane == 0) {
      erange[0] = nlo;
      erange[1] = nhi;
    }
  }
  __syncthreads();
  const int e_lo = erange[0], n_sel = erange[1] - erange[0];
  const bool diag = t >= c_lo && t < c_hi;
  const int upb = p.block / 16;  // 16-token units per block
  const int n_units = n_sel * upb + (diag ? (pos - t * p.block) / 16 + 1 : 0);
  const float qk_scale = rsqrtf((float)D) * kLog2e;
  const T* kg = static_cast<const T*>(p.k.data) + (int64_t)b * p.k.sb + (int64_t)g * p.k.sh;
  const T* vg = static_cast<const T*>(p.v.data) + (int64_t)b * p.v.sb + (int64_t)g * p.v.sh;

  float qv[G][DL];
  {
    const T* q = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb;
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < DL; ++e)
        qv[h][e] = Elt<T>::load1(q + (int64_t)(g * G + h) * p.q.sh + lane * DL + e) * qk_scale;
  }
  auto load_row = [&](const T* base, int64_t ss, int tok, float* f) {  // this lane's DL values of a cache row
    const T* src = base + (int64_t)(tok - p.tok_lo) * ss + lane * DL;
    float f8[8];
    if constexpr (DL == 4) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
      Elt<T>::to_float(make_uint4(raw.x, raw.y, 0u, 0u), f8);
    } else {
      const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(src));
      Elt<T>::to_float(make_uint4(raw, 0u, 0u, 0u), f8);
    }
#pragma unroll
    for (int e = 0; e < DL; ++e) f[e] = f8[e];
  };

  float m[G], o[G][DL], lown[NVL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = kNegInf;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[h][e] = 0.f;
  }
#pragma unroll
  for (int j = 0; j < NVL; ++j) lown[j] = 0.f;

  for (int u = warp; u < n_units; u += W) {
    int tok0;
    float bias;
    if (u < n_sel * upb) {
      const int e = e_lo + u / upb;
      tok0 = idx[e] * p.block + (u % upb) * 16;
      bias = p.sigma * logp[e] * kLog2e;
    } else {
      tok0 = t * p.block + (u - n_sel * upb) * 16;
      bias = beta * kLog2e;
    }
    float v[NV];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
      float kf[DL];
      if (tok0 + tt <= pos) {
        load_row(kg, p.k.ss, tok0 + tt, kf);
      } else {
#pragma unroll
        for (int e = 0; e < DL; ++e) kf[e] = 0.f;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) a = fmaf(qv[h][e], kf[e], a);
        v[tt * G + h] = a;
      }
    }
    warp_transpose_reduce<NV>(v, lane);
    // lane holds token lane/2; heads (lane&1)*GH + j (G >= 2) or head 0
    const bool valid = tok0 + (lane >> 1) <= pos;
    float sl[NVL], mx[NVL];
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
      sl[j] = valid ? v[j] + bias : kNegInf;
      mx[j] = sl[j];
#pragma unroll
      for (int off = 2; off <= 16; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], off));
    }
    float mu[G], sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float th = __shfl_sync(0xffffffffu, mx[h % GH], G >= 2 ? h / GH : 0);
      const float mn = fmaxf(m[h], th);
      mu[h] = mn == kNegInf ? 0.f : mn;
      sc[h] = exp2f(m[h] - mu[h]);
      m[h] = mn;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[h][e] *= sc[h];
    }
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
      const int hd = G >= 2 ? (lane & 1) * GH + j : 0;
      float muj = mu[j], scj = sc[j];
      if constexpr (G >= 2) {
        muj = (lane & 1) ? mu[GH + j] : mu[j];
        scj = (lane & 1) ? sc[GH + j] : sc[j];
      }
      const float pj = exp2f(sl[j] - muj);
      lown[j] = lown[j] * scj + pj;
      pbuf[warp][(lane >> 1) * G + hd] = pj;
    }
    __syncwarp();
#pragma unroll 4
    for (int tt = 0; tt < 16; ++tt) {
      if (tok0 + tt > pos) break;
      float vf[DL];
      load_row(vg, p.v.ss, tok0 + tt, vf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ph = pbuf[warp][tt * G + h];
#pragma unroll
        for (int e = 0; e < DL; ++e) o[h][e] = fmaf(ph, vf[e], o[h][e]);
      }
    }
    __syncwarp();
  }

  // merge the warps: l per head over the 16 lanes of its parity
#pragma unroll
  for (int j = 0; j < NVL; ++j)
#pragma unroll
    for (int off = 2; off <= 16; off <<= 1) lown[j] += __shfl_xor_sync(0xffffffffu, lown[j], off);
  if (lane < 2) {
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
      if (G >= 2) {
        lbuf[warp][lane * GH + j] = lown[j];
      } else if (lane == 0) {
        lbuf[warp][0] = lown[0];
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) mbuf[warp][h] = m[h];
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL; ++e) obuf[warp][h][lane * DL + e] = o[h][e];
  __syncthreads();
  for (int i = tid; i < G * D; i += W * 32) {
    const int h = i / D, e = i % D;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, mbuf[w][h]);
    const float Mu = M == kNegInf ? 0.f : M;
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = exp2f(mbuf[w][h] - Mu);
      acc += f * obuf[w][h][e];
      lsum += f * lbuf[w][h];
    }
    float* part = p.part + ((int64_t)b * p.H + g * G + h) * (D + 2);
    part[e] = acc;
    if (e == 0) {
      part[D] = M;
      part[D + 1] = lsum;
    }
  }
}

// Log-sum-exp merge of the shards' partials into the output.
template <typename T>
__global__ void __launch_bounds__(128) cp_merge_kernel(const float* parts, int n_parts, int B, int H, int D,
                                                       View out) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t stride = (int64_t)B * H * (D + 2);
  const float* p0 = parts + ((int64_t)b * H + h) * (D + 2);
  float M = kNegInf;
  for (int r = 0; r < n_parts; ++r) M = fmaxf(M, p0[r * stride + D]);
  const float Mu = M == kNegInf ? 0.f : M;
  T* dst = static_cast<T*>(const_cast<void*>(out.data)) + (int64_t)b * out.sb + (int64_t)h * out.sh;
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float acc = 0.f, lsum = 0.f;
    for (int r = 0; r < n_parts; ++r) {
      const float* pr = p0 + r * stride;
      const float f = exp2f(pr[D] - Mu);
      acc += f * pr[e];
      lsum += f * pr[D + 1];
    }
    Elt<T>::store1(dst + e, lsum > 0.f ? acc / lsum : 0.f);
  }
}

// ------------------------------------------------------------------ combine
template <typename T, int D>
__global__ void __launch_bounds__(256) combine_decode_kernel(DecodeParams p) {
  const int b = blockIdx.y, g = blockIdx.x;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int n_it = (p.cnt[bg] + 1 + p.chunk_blocks - 1) / p.chunk_blocks;
  const int64_t base = p.pair_base[bg];
  T* out = static_cast<T*>(const_cast<void*>(p.out.data)) + (int64_t)b * p.out.sb;
  for (int i = threadIdx.x; i < p.G * D; i += blockDim.x) {
    const int h = i / D, e = i % D;
    float M = kNegInf;
    for (int k = 0; k < n_it; ++k) M = fmaxf(M, p.part_ml[((base + k) * p.G + h) * 2]);
    const float Mu = M == kNegInf ? 0.f : M;
    float acc = 0.f, lsum = 0.f;
    for (int k = 0; k < n_it; ++k) {
      const float f = exp2f(p.part_ml[((base + k) * p.G + h) * 2] - Mu);
      acc += f * p.part_o[((base + k) * p.G + h) * D + e];
      lsum += f * p.part_ml[((base + k) * p.G + h) * 2 + 1];
    }
    Elt<T>::store1(out + (int64_t)(g * p.G + h) * p.out.sh + e, lsum > 0.f ? acc / lsum : 0.f);
  }
}

// Context parallelism on the split-KV path: the part of each (sequence, KV
// head)'s ascending list that falls in this shard's blocks [block_lo,
// block_hi) is a contiguous entry range; with the diagonal block when the
// shard holds it, it is cut into work items of chunk_blocks entries as in
// the regular decode (one warp per (b, g)).
__global__ void __launch_bounds__(256) shard_items_kernel(DecodeParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bg = (int64_t)blockIdx.x * 8 + warp;
  if (bg >= (int64_t)p.B * p.Hkv) return;
  const int b = (int)(bg / p.Hkv);
  const int L = clamp_len(p.seqlens, b, p.Lmax, nullptr);
  const int t = (L - 1) / p.block;
  const int block_lo = p.tok_lo / p.block, block_hi = (p.tok_lo + p.tok_n) / p.block;
  const int cnt = min(max(p.cnt[bg], 0), (int)p.t_cap);
  const int32_t* idx = p.idx + bg * p.t_cap;
  int below_lo = 0, below_hi = 0;  // entries before the shard's first block / past its last
  for (int e = lane; e < cnt; e += 32) {
    const int c = idx[e];
    below_lo += c < block_lo ? 1 : 0;
    below_hi += c < block_hi ? 1 : 0;
  }
  below_lo = warp_sum_i(below_lo);
  below_hi = warp_sum_i(below_hi);
  if (lane == 0) {
    const int diag = (t >= block_lo && t < block_hi) ? 1 : 0;
    const int n_entries = below_hi - below_lo + diag;
    const int n_it = (n_entries + p.chunk_blocks - 1) / p.chunk_blocks;
    const int base = n_it > 0 ? atomicAdd(p.n_items, n_it) : 0;
    p.pair_base[bg] = base;
    p.shard[4 * bg] = below_lo;
    p.shard[4 * bg + 1] = below_hi;
    p.shard[4 * bg + 2] = diag;
    p.shard[4 * bg + 3] = n_it;
    for (int k = 0; k < n_it; ++k) {
      p.items[2 * (base + k)] = (int32_t)bg;
      p.items[2 * (base + k) + 1] = k;
    }
  }
}

// The shard's per-head partial of each (b, g): log-sum-exp merge of its
// items' partials, left unnormalised for the merge across shards (o relative
// to the reference max m, m in log2 units, l); no items: m = -inf, l = 0.
template <int D>
__global__ void __launch_bounds__(256) combine_partial_kernel(DecodeParams p) {
  const int b = blockIdx.y, g = blockIdx.x;
  const int64_t bg = (int64_t)b * p.Hkv + g;
  const int n_it = p.shard[4 * bg + 3];
  const int64_t base = p.pair_base[bg];
  for (int i = threadIdx.x; i < p.G * D; i += blockDim.x) {
    const int h = i / D, e = i % D;
    float M = kNegInf;
    for (int k = 0; k < n_it; ++k) M = fmaxf(M, p.part_ml[((base + k) * p.G + h) * 2]);
    const float Mu = M == kNegInf ? 0.f : M;
    float acc = 0.f, lsum = 0.f;
    for (int k = 0; k < n_it; ++k) {
      const float f = exp2f(p.part_ml[((base + k) * p.G + h) * 2] - Mu);
      acc += f * p.part_o[((base + k) * p.G + h) * D + e];
      lsum += f * p.part_ml[((base + k) * p.G + h) * 2 + 1];
    }
    float* part = p.part + ((int64_t)b * p.H + g * p.G + h) * (D + 2);
    part[e] = acc;
    if (e == 0) {
      part[D] = M;
      part[D + 1] = lsum;
    }
  }
}

template <typename T, int D, int G>
cudaError_t launch_route_t(const DecodeParams& p, cudaStream_t stream) {
  dim3 grid((unsigned)((p.t_cap + 63) / 64), p.Hkv, p.B);
  score_decode_kernel<T, D, G><<<grid, 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)G * p.t_cap * sizeof(float);
  e = cudaFuncSetAttribute(entmax_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  entmax_decode_kernel<<<dim3(p.Hkv, p.B), 256, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t launch_attend_t(const DecodeParams& p, int num_sms, cudaStream_t stream, bool partial = false) {
  const size_t smem =
      (size_t)2 * kDStages * kStep * D * sizeof(T) + (size_t)(2 * kWarps * G + kWarps * G * D) * sizeof(float);
  auto kern = attend_decode_mma_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarps * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  kern<<<num_sms * per_sm, kWarps * 32, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (partial)
    combine_partial_kernel<D><<<dim3(p.Hkv, p.B), 256, 0, stream>>>(p);
  else
    combine_decode_kernel<T, D><<<dim3(p.Hkv, p.B), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t route_d(const DecodeParams& p, cudaStream_t s) {
  switch (p.G) {
    case 1: return launch_route_t<T, D, 1>(p, s);
    case 2: return launch_route_t<T, D, 2>(p, s);
    case 4: return launch_route_t<T, D, 4>(p, s);
    default: return launch_route_t<T, D, 8>(p, s);
  }
}
template <typename T, int D>
cudaError_t attend_d(const DecodeParams& p, int n, cudaStream_t s, bool partial = false) {
  switch (p.G) {
    case 1: return launch_attend_t<T, D, 1>(p, n, s, partial);
    case 2: return launch_attend_t<T, D, 2>(p, n, s, partial);
    case 4: return launch_attend_t<T, D, 4>(p, n, s, partial);
    default: return launch_attend_t<T, D, 8>(p, n, s, partial);
  }
}

}  // namespace

int64_t decode_max_items(int64_t B, int64_t Hkv, int64_t t_cap, int chunk_blocks) {
  return B * Hkv * ((t_cap + 1 + chunk_blocks - 1) / chunk_blocks);
}

cudaError_t launch_decode_route(const DecodeParams& p, cudaStream_t stream) {
  if (p.D == 128) {
    if (p.dtype == 0) return route_d<float, 128>(p, stream);
    if (p.dtype == 1) return route_d<__half, 128>(p, stream);
    return route_d<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 0) return route_d<float, 64>(p, stream);
  if (p.dtype == 1) return route_d<__half, 64>(p, stream);
  return route_d<__nv_bfloat16, 64>(p, stream);
}

cudaError_t launch_decode_attend(const DecodeParams& p, int num_sms, cudaStream_t stream) {
  if (p.dtype == 0) return cudaErrorInvalidValue;  // fp32 decode is not supported
  if (p.D == 128) {
    if (p.dtype == 1) return attend_d<__half, 128>(p, num_sms, stream);
    return attend_d<__nv_bfloat16, 128>(p, num_sms, stream);
  }
  if (p.dtype == 1) return attend_d<__half, 64>(p, num_sms, stream);
  return attend_d<__nv_bfloat16, 64>(p, num_sms, stream);
}

namespace {
template <typename T, int D>
cudaError_t cp_scores_d(const DecodeParams& p, cudaStream_t s) {
  dim3 grid((unsigned)((p.t_cap + 63) / 64), p.Hkv, p.B);
  switch (p.G) {
    case 1: score_decode_kernel<T, D, 1><<<grid, 256, 0, s>>>(p); break;
    case 2: score_decode_kernel<T, D, 2><<<grid, 256, 0, s>>>(p); break;
    case 4: score_decode_kernel<T, D, 4><<<grid, 256, 0, s>>>(p); break;
    default: score_decode_kernel<T, D, 8><<<grid, 256, 0, s>>>(p); break;
  }
  return cudaGetLastError();
}
template <typename T, int D>
cudaError_t cp_attend_d(const DecodeParams& p, cudaStream_t s) {
  dim3 grid(p.Hkv, p.B);
  switch (p.G) {
    case 1: attend_shard_kernel<T, D, 1><<<grid, 128, 0, s>>>(p); break;
    case 2: attend_shard_kernel<T, D, 2><<<grid, 128, 0, s>>>(p); break;
    case 4: attend_shard_kernel<T, D, 4><<<grid, 128, 0, s>>>(p); break;
    default: attend_shard_kernel<T, D, 8><<<grid, 128, 0, s>>>(p); break;
  }
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_cp_scores(const DecodeParams& p, cudaStream_t stream) {
  if (p.D == 128) return p.dtype == 1 ? cp_scores_d<__half, 128>(p, stream) : cp_scores_d<__nv_bfloat16, 128>(p, stream);
  return p.dtype == 1 ? cp_scores_d<__half, 64>(p, stream) : cp_scores_d<__nv_bfloat16, 64>(p, stream);
}

cudaError_t launch_cp_lists(const DecodeParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.G * p.t_cap * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(entmax_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  entmax_decode_kernel<<<dim3(p.Hkv, p.B), 256, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cp_attend(const DecodeParams& p, cudaStream_t stream) {
  if (p.D == 128) return p.dtype == 1 ? cp_attend_d<__half, 128>(p, stream) : cp_attend_d<__nv_bfloat16, 128>(p, stream);
  return p.dtype == 1 ? cp_attend_d<__half, 64>(p, stream) : cp_attend_d<__nv_bfloat16, 64>(p, stream);
}

cudaError_t launch_cp_attend_mma(const DecodeParams& p, int num_sms, cudaStream_t stream) {
  if (p.dtype == 0 || !p.shard) return cudaErrorInvalidValue;
  const int64_t n_bg = (int64_t)p.B * p.Hkv;
  shard_items_kernel<<<(unsigned)((n_bg + 7) / 8), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.D == 128) {
    if (p.dtype == 1) return attend_d<__half, 128>(p, num_sms, stream, true);
    return attend_d<__nv_bfloat16, 128>(p, num_sms, stream, true);
  }
  if (p.dtype == 1) return attend_d<__half, 64>(p, num_sms, stream, true);
  return attend_d<__nv_bfloat16, 64>(p, num_sms, stream, true);
}

cudaError_t launch_cp_merge(const float* parts, int n_parts, int B, int H, int D, const View& out, int dtype,
                            cudaStream_t stream) {
  dim3 grid(H, B);
  if (dtype == 1)
    cp_merge_kernel<__half><<<grid, 128, 0, stream>>>(parts, n_parts, B, H, D, out);
  else
    cp_merge_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(parts, n_parts, B, H, D, out);
  return cudaGetLastError();
}

}  // namespace dash
