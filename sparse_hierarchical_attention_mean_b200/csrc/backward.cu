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
// Four kernels, all on the forward's lists (the union of a query block's
// lists is rebuilt here):
//   bwd_row    one CTA per (query block, head); warp w owns 16 rows.  One
//              pass over the 64-key chunks of the union of the rows'
//              selected blocks and the diagonal block, with each row's
//              log-sum-exp from the forward's stage-2 kernel: P, dP = dout
//              V^T, dS = P (dP - D) and dq = dS K / sqrt(d), plus each row's
//              d log p_bar of every selected block (the row sum of dS over the
//              block).  All three products are warp-level MMAs (m16n8k16,
//              fp32 accumulate); dS is the accumulator re-packed as the A
//              operand.
//   bwd_route  one CTA per (row, KV head): the entmax vector-Jacobian
//              product per head from the recomputed scores and the
//              forward's thresholds, and dq += gamma dz S.
//   bwd_key    one CTA per (key block, KV head); warp w owns 16 keys.  Walks
//              the query blocks whose union holds the block (and its own
//              diagonal block), finds each row's list entry by binary search,
//              and accumulates dv = P^T dout and dk = dS^T q / sqrt(d) in
//              registers, and the summary gradient ds = gamma sum dz q.  Its
//              epilogue adds the stage-0 term ds W_s^T / |c| to every key of
//              the block and stores the block mean for dW_s.
//   bwd_ws     dW_s = sum over blocks of kbar^T ds.
// Tiles in shared memory are XOR-swizzled by row (mma_sync.cuh) and filled by
// cp.async with zero fill past the sequence end; bwd_row and bwd_key
// double-buffer what they stream (the next K/V chunk, the next (head, row
// chunk) item with its rows' statistics) so the copies overlap the MMAs.
#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"

namespace dash {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kKeyChunk = 64;  // keys per step of bwd_row

// rows [0, n_rows) of a [n_rows][D] tile from `g` (row stride `stride`
// elements); rows >= n_valid are zero-filled.  Requires n_valid >= 1.
template <typename T, int D>
__device__ __forceinline__ void load_rows(T* sm, const T* g, int64_t stride, int n_valid, int n_rows, int tid,
                                          int nth) {
  constexpr int NCH = D / 8;
  for (int i = tid; i < n_rows * NCH; i += nth) {
    const int r = i / NCH, c = i % NCH;
    const bool ok = r < n_valid;
    cp_async16(sm + r * D + ((c ^ (r & 7)) << 3), g + (int64_t)(ok ? r : 0) * stride + c * 8, ok);
  }
}

// A fragment (16 rows from `row0`, d columns 16 kk .. 16 kk + 15) of a swizzled tile.
template <typename T, int D>
__device__ __forceinline__ void load_a(uint32_t base, int row0, int kk, int lane, uint32_t* a) {
  const int r = row0 + (lane & 15);
  const int c = 2 * kk + (lane >> 4);
  ldsm_x4(base + (uint32_t)((r * D + ((c ^ (r & 7)) << 3)) * sizeof(T)), a);
}

// acc[NP * 2][4] = A (16 rows of tile `abase` from a_row0) * B^T, B = rows
// 0 .. 16 NP - 1 of tile `bbase`; contraction over D.
template <typename T, int D, int NP>
__device__ __forceinline__ void tile_abt(uint32_t abase, int a_row0, uint32_t bbase, int lane, float (*acc)[4]) {
#pragma unroll
  for (int n = 0; n < 2 * NP; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int m = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    load_a<T, D>(abase, a_row0, kk, lane, a);
#pragma unroll
    for (int np = 0; np < NP; ++np) {
      const int tok = np * 16 + (m >> 1) * 8 + rr;
      const int c = 2 * kk + (m & 1);
      uint32_t bf[4];
      ldsm_x4(bbase + (uint32_t)((tok * D + ((c ^ (tok & 7)) << 3)) * sizeof(T)), bf);
      mma16816<T>(acc[2 * np], a, bf[0], bf[1]);
      mma16816<T>(acc[2 * np + 1], a, bf[2], bf[3]);
    }
  }
}

// out[D/8][4] += X (16 x 16 KSTEP, given as accumulator fragments x[2 KSTEP][4])
// * B, B = rows 0 .. 16 KSTEP - 1 of tile `bbase` ([rows][D]).
template <typename T, int D, int KSTEP>
__device__ __forceinline__ void tile_xb(const float (*x)[4], uint32_t bbase, int lane, float (*out)[4]) {
  const int m = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int ks = 0; ks < KSTEP; ++ks) {
    const uint32_t a[4] = {pack2<T>(x[2 * ks][0], x[2 * ks][1]), pack2<T>(x[2 * ks][2], x[2 * ks][3]),
                           pack2<T>(x[2 * ks + 1][0], x[2 * ks + 1][1]),
                           pack2<T>(x[2 * ks + 1][2], x[2 * ks + 1][3])};
    const int tok = ks * 16 + (m & 1) * 8 + rr;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      const int c = 2 * j + (m >> 1);
      uint32_t bf[4];
      ldsm_x4_t(bbase + (uint32_t)((tok * D + ((c ^ (tok & 7)) << 3)) * sizeof(T)), bf);
      mma16816<T>(out[2 * j], a, bf[0], bf[1]);
      mma16816<T>(out[2 * j + 1], a, bf[2], bf[3]);
    }
  }
}

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(kFull, x, 1);
  return x + __shfl_xor_sync(kFull, x, 2);
}

// prior of the diagonal block, log2 units: sigma * log(1/N), 0 when N = 0
__device__ __forceinline__ float diag_bias2(float sigma, int n_cand) {
  return n_cand > 0 ? sigma * logf(1.0f / (float)n_cand) * kLog2e : 0.f;
}

// ------------------------------------------------------------------ bwd_row
template <typename T, int D, int BLK>
__global__ void __launch_bounds__(2 * BLK) bwd_row_kernel(BwdParams p) {
  constexpr int NW = BLK / 16, NTH = NW * 32;
  constexpr int SPB = BLK / kKeyChunk;  // chunks per block
  constexpr int NT = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  T* Qs = reinterpret_cast<T*>(smem);  // [BLK][D]
  T* dOs = Qs + BLK * D;               // [BLK][D]
  T* Ks = dOs + BLK * D;               // [2][64][D] (double buffer)
  T* Vs = Ks + 2 * kKeyChunk * D;      // [2][64][D]
  float* Dsm = reinterpret_cast<float*>(Vs + 2 * kKeyChunk * D);  // [BLK] dout . out
  uint32_t* um = reinterpret_cast<uint32_t*>(Dsm + BLK);      // [n_words] union bitmap
  int32_t* ulist = reinterpret_cast<int32_t*>(um + p.n_words);  // [t_cap + 1] union, then the diagonal
  __shared__ int nu_s;

  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / p.G, hh = h - g * p.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int S = p.S;
  const int64_t tc = p.t_cap;
  const int row0 = t * BLK;
  const int nrows = min(BLK, S - row0);
  const int64_t rowbase = ((int64_t)b * p.Hkv + g) * S;

  // union of the rows' selected blocks
  for (int w = tid; w < p.n_words; w += NTH) um[w] = 0u;
  __syncthreads();
  for (int r = warp; r < nrows; r += NW) {
    const int n = p.cnt[rowbase + row0 + r];
    const int32_t* list = p.idx + (rowbase + row0 + r) * tc;
    for (int e = lane; e < n; e += 32) {
      const int c = list[e];
      if ((unsigned)c < (unsigned)tc) atomicOr(&um[c >> 5], 1u << (c & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < p.n_words; w0 += 32) {
      const uint32_t word = w0 + lane < p.n_words ? um[w0 + lane] : 0u;
      const int nb = __popc(word);
      int incl = nb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = base + incl - nb;
      for (uint32_t wd = word; wd; wd &= wd - 1) ulist[pos++] = (w0 + lane) * 32 + (__ffs(wd) - 1);
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) {
      ulist[base] = t;
      nu_s = base;
    }
  }
  if (hh == 0) {
    uint32_t* gm = p.umask + ((int64_t)b * p.Hkv * p.n_qblocks + (int64_t)g * p.n_qblocks + t) * p.n_words;
    for (int w = tid; w < p.n_words; w += NTH) gm[w] = um[w];
  }

  // this head's Q and dout rows; D = dout . out per row
  {
    const T* qg = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb + (int64_t)row0 * p.q.ss + (int64_t)h * p.q.sh;
    const T* dg = static_cast<const T*>(p.dout.data) + (int64_t)b * p.dout.sb + (int64_t)row0 * p.dout.ss +
                  (int64_t)h * p.dout.sh;
    load_rows<T, D>(Qs, qg, p.q.ss, nrows, BLK, tid, NTH);
    load_rows<T, D>(dOs, dg, p.dout.ss, nrows, BLK, tid, NTH);
    cp_async_commit();
    const T* og = static_cast<const T*>(p.o.data) + (int64_t)b * p.o.sb + (int64_t)row0 * p.o.ss + (int64_t)h * p.o.sh;
    for (int r = warp; r < BLK; r += NW) {
      float acc = 0.f;
      if (r < nrows) {
        for (int c = lane; c < D; c += 32)
          acc = fmaf(Elt<T>::load1(og + (int64_t)r * p.o.ss + c), Elt<T>::load1(dg + (int64_t)r * p.dout.ss + c), acc);
        acc = warp_sum(acc);
        if (lane == 0) p.dd[((int64_t)b * p.H + h) * S + row0 + r] = acc;
      }
      if (lane == 0) Dsm[r] = acc;
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  const int nu = nu_s;
  const int nchunks = (nu + 1) * SPB;
  const float sc = rsqrtf((float)D) * kLog2e;
  const int n_cand = p.causal ? t : p.n_qblocks - 1;
  const float beta2 = diag_bias2(p.sigma, n_cand);
  const int ra = warp * 16 + gq, rb = ra + 8;
  const bool va = ra < nrows, vb = rb < nrows;
  const int pa = row0 + ra, pb = row0 + rb;
  const int cnt_a = va ? p.cnt[rowbase + pa] : 0, cnt_b = vb ? p.cnt[rowbase + pb] : 0;
  const int32_t* list_a = p.idx + (rowbase + (va ? pa : row0)) * tc;
  const int32_t* list_b = p.idx + (rowbase + (vb ? pb : row0)) * tc;
  const float* lp_a = p.logp + (rowbase + (va ? pa : row0)) * tc;
  const float* lp_b = p.logp + (rowbase + (vb ? pb : row0)) * tc;
  const T* kg = static_cast<const T*>(p.k.data) + (int64_t)b * p.k.sb + (int64_t)g * p.k.sh;
  const T* vg = static_cast<const T*>(p.v.data) + (int64_t)b * p.v.sb + (int64_t)g * p.v.sh;
  const uint32_t qs_b = smem_u32(Qs), do_b = smem_u32(dOs), ks_b = smem_u32(Ks), vs_b = smem_u32(Vs);

  // bias (log2 units) of rows a and b for block c; entries ea/eb of c in the
  // rows' lists (-1: not selected); cursors move past c after its last chunk
  int cur_a = 0, cur_b = 0;
  auto row_bias = [&](int c, bool diag, int sub, float& ba, float& bb, int& ea, int& eb) {
    if (diag) {
      ba = va ? beta2 : kNegInf;
      bb = vb ? beta2 : kNegInf;
      ea = eb = -1;
      return;
    }
    ea = (cur_a < cnt_a && list_a[cur_a] == c) ? cur_a : -1;
    eb = (cur_b < cnt_b && list_b[cur_b] == c) ? cur_b : -1;
    ba = ea >= 0 ? p.sigma * lp_a[ea] * kLog2e : kNegInf;
    bb = eb >= 0 ? p.sigma * lp_b[eb] * kLog2e : kNegInf;
    if (sub == SPB - 1) {
      cur_a += ea >= 0;
      cur_b += eb >= 0;
    }
  };
  // logits of the lane's 32 (row, key) pairs in place, log2 units, -inf when masked
  auto logits = [&](float (*s)[4], int key0, bool diag, float ba, float bb) {
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + n * 8 + 2 * tq + (e & 1);
        const int row = e < 2 ? pa : pb;
        const bool ok = key < S && (!diag || !p.causal || key <= row);
        s[n][e] = ok ? fmaf(s[n][e], sc, e < 2 ? ba : bb) : kNegInf;
      }
  };

  // chunks with keys to process (the others are past the sequence end or,
  // on the causal diagonal, past every row of the block)
  auto chunk_ok = [&](int ch) -> bool {
    const int bi = ch / SPB, sub = ch - bi * SPB;
    const int key0 = ulist[bi] * BLK + sub * kKeyChunk;
    return !(key0 >= S || (bi == nu && p.causal && key0 > row0 + nrows - 1));
  };
  auto next_ok = [&](int ch) -> int {
    while (ch < nchunks && !chunk_ok(ch)) ++ch;
    return ch;
  };
  // K (and V) rows of chunk ch into buffer buf
  auto issue = [&](int ch, int buf, bool with_v) {
    if (ch < nchunks) {
      const int bi = ch / SPB, sub = ch - bi * SPB;
      const int key0 = ulist[bi] * BLK + sub * kKeyChunk;
      const int nk = min(kKeyChunk, S - key0);
      load_rows<T, D>(Ks + buf * kKeyChunk * D, kg + (int64_t)key0 * p.k.ss, p.k.ss, nk, kKeyChunk, tid, NTH);
      if (with_v)
        load_rows<T, D>(Vs + buf * kKeyChunk * D, vg + (int64_t)key0 * p.v.ss, p.v.ss, nk, kKeyChunk, tid, NTH);
    }
    cp_async_commit();
  };
  constexpr uint32_t kBufBytes = kKeyChunk * D * sizeof(T);

  // each row's log-sum-exp (log2 units) comes from the forward's stage-2 kernel
  int buf = 0;
  const float lse_a = va ? p.lse[((int64_t)b * p.H + h) * S + pa] : 0.f;
  const float lse_b = vb ? p.lse[((int64_t)b * p.H + h) * S + pb] : 0.f;
  const float d_a = Dsm[ra], d_b = Dsm[rb];

  // pass 2: dS, dq and d log p_bar, with the same prefetch of K and V
  float dq[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
  float dl_a = 0.f, dl_b = 0.f;
  float* dz_a = p.dz + (rowbase + (va ? pa : row0)) * tc * p.G + hh;
  float* dz_b = p.dz + (rowbase + (vb ? pb : row0)) * tc * p.G + hh;
  issue(next_ok(0), 0, true);
  for (int ch = 0; ch < nchunks; ++ch) {
    const int bi = ch / SPB, sub = ch - bi * SPB;
    const int c = ulist[bi];
    const bool diag = bi == nu;
    const int key0 = c * BLK + sub * kKeyChunk;
    float ba, bb;
    int ea, eb;
    row_bias(c, diag, sub, ba, bb, ea, eb);
    if (chunk_ok(ch)) {
      __syncthreads();
      issue(next_ok(ch + 1), buf ^ 1, true);
      cp_async_wait<1>();
      __syncthreads();
      const uint32_t kb = ks_b + buf * kBufBytes, vb_ = vs_b + buf * kBufBytes;
      float s[8][4], dp[8][4];
      tile_abt<T, D, 4>(qs_b, warp * 16, kb, lane, s);
      tile_abt<T, D, 4>(do_b, warp * 16, vb_, lane, dp);
      logits(s, key0, diag, ba, bb);
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pr = exp2f(s[n][e] - (e < 2 ? lse_a : lse_b));  // 0 where masked
          const float dsv = pr * (dp[n][e] - (e < 2 ? d_a : d_b));
          s[n][e] = dsv;
          if (e < 2) dl_a += dsv;
          else dl_b += dsv;
        }
      tile_xb<T, D, 4>(s, kb, lane, dq);
      buf ^= 1;
    }
    if (!diag && sub == SPB - 1) {
      dl_a = quad_sum(dl_a);
      dl_b = quad_sum(dl_b);
      if (tq == 0) {
        if (ea >= 0) dz_a[(int64_t)ea * p.G] = p.sigma * dl_a;
        if (eb >= 0) dz_b[(int64_t)eb * p.G] = p.sigma * dl_b;
      }
    }
    if (sub == SPB - 1) dl_a = dl_b = 0.f;
  }
  cp_async_wait<0>();

  const float qsc = rsqrtf((float)D);
  float* dqg = static_cast<float*>(const_cast<void*>(p.dq.data)) + (int64_t)b * p.dq.sb + (int64_t)h * p.dq.sh;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int col = n * 8 + 2 * tq;
    if (va) *reinterpret_cast<float2*>(dqg + (int64_t)pa * p.dq.ss + col) = make_float2(dq[n][0] * qsc, dq[n][1] * qsc);
    if (vb) *reinterpret_cast<float2*>(dqg + (int64_t)pb * p.dq.ss + col) = make_float2(dq[n][2] * qsc, dq[n][3] * qsc);
  }
}

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

template <typename T, int D, int BLK>
cudaError_t launch_typed(const BwdParams& p, cudaStream_t stream) {
  const size_t row_smem = (size_t)(2 * BLK * D + 4 * kKeyChunk * D) * sizeof(T) + BLK * 4 +
                          (size_t)(p.n_words + p.t_cap + 1) * 4;
  cudaError_t e = cudaFuncSetAttribute(bwd_row_kernel<T, D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)row_smem);
  if (e != cudaSuccess) return e;
  bwd_row_kernel<T, D, BLK><<<dim3(p.n_qblocks, p.H, p.B), 2 * BLK, row_smem, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

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
  if (p.D == 128) return p.block == 128 ? launch_typed<T, 128, 128>(p, stream) : launch_typed<T, 128, 64>(p, stream);
  return p.block == 128 ? launch_typed<T, 64, 128>(p, stream) : launch_typed<T, 64, 64>(p, stream);
}

}  // namespace

cudaError_t launch_bwd(const BwdParams& p, cudaStream_t stream) {
  if (p.dtype == 1) return launch_dtype<__half>(p, stream);
  return launch_dtype<__nv_bfloat16>(p, stream);
}

}  // namespace dash
