// Stage 2 for prefill: prior-induced sparse softmax over the selected blocks.
//
// "Stage 2: prior-induced sparse softmax" of the DashAttention technical
// summary: softmax is the maximiser of <p, l> - KL(p || u); replacing the
// uniform reference u by a prior g built from the routing weights gives
// softmax(l + log g), and g = 0 on blocks with zero routing mass masks them.
// Near-diagonal chunks have no summary and are handled by a separate branch
// (here: the query's own block, always included, with the uniform-baseline
// prior log(1/N) and a causal mask).  The implementation walks the active
// chunks and adds the routing bias to the logits before the softmax.
//
// Tensor-core kernel (f16/bf16, fp32 accumulation): one CTA owns a tile of
// P positions x G heads = 16 * NW rows of one KV group, so every K/V block
// fetched serves all G heads.  It iterates over the union of the tile's
// selected blocks (ascending) and then the diagonal block, 64 tokens per
// step, with K/V double-buffered through cp.async.  Each row walks its own
// ascending list to find its bias for the current block (-inf if the row
// did not select it).  Online softmax in the log2 domain.
//
// fp32 inputs use a CUDA-core kernel with one warp per (position, head) row.
#include "common.cuh"
#include "internal.h"

namespace dash {
namespace {

// ---------------------------------------------------------------- mma.sync helpers
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

template <typename T>
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1);
template <>
__device__ __forceinline__ void mma16816<__nv_bfloat16>(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma16816<__half>(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Swizzled [rows][D] tile of 16-bit elements: 16-byte chunk c of row r sits at
// chunk c ^ (r & 7), which makes ldmatrix reads conflict-free.
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

constexpr int kKV = 64;  // tokens per step

// Row state for the per-row list walk.
struct RowList {
  const int32_t* idx;
  const float* logp;
  int cnt, cur, next;
  __device__ __forceinline__ void init(const int32_t* i, const float* l, int n) {
    idx = i;
    logp = l;
    cnt = n;
    cur = 0;
    next = n > 0 ? i[0] : 0x7fffffff;
  }
  // bias (natural log) for block c; advances past c
  __device__ __forceinline__ float bias_for(int c) {
    float bias = kNegInf;
    if (next == c) {
      bias = logp[cur];
      ++cur;
      next = cur < cnt ? idx[cur] : 0x7fffffff;
    }
    return bias;
  }
};

template <typename T, int D, int NW>
__global__ void __launch_bounds__(NW * 32) sparse_prefill_mma_kernel(SparseParams p) {
  constexpr int ROWS = 16 * NW;
  constexpr int NCH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  T* Qs = reinterpret_cast<T*>(smem_raw);
  T* Ks = Qs + ROWS * D;      // [2][kKV][D]
  T* Vs = Ks + 2 * kKV * D;   // [2][kKV][D]

  const int b = blockIdx.z, g = blockIdx.y, tile = blockIdx.x;
  const int G = p.G;
  const int P = p.tile_pos;
  const int pos0 = tile * P;
  const int t = pos0 / p.block;
  const int T_ = (p.S + p.block - 1) / p.block;
  const int N = p.causal ? t : T_ - 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bg = (int64_t)b * p.Hkv + g;

  const T* qg = static_cast<const T*>(p.q.data) + (int64_t)b * p.q.sb;
  const T* kg = static_cast<const T*>(p.k.data) + (int64_t)b * p.k.sb + (int64_t)g * p.k.sh;
  const T* vg = static_cast<const T*>(p.v.data) + (int64_t)b * p.v.sb + (int64_t)g * p.v.sh;

  // ---- Q tile -> shared
  for (int i = tid; i < ROWS * NCH; i += NW * 32) {
    const int r = i / NCH, c = i % NCH;
    const int pos = pos0 + r / G, head = g * G + r % G;
    const bool ok = pos < p.S && r / G < P;
    const T* src = qg + (int64_t)(ok ? pos : 0) * p.q.ss + (int64_t)head * p.q.sh + c * 8;
    cp_async16(Qs + swz<D>(r, c), src, ok);
  }
  cp_async_commit();

  // ---- work list: union blocks (per 64-token half) then the diagonal block
  const int spb = p.block / kKV;
  const int32_t* ulist = p.ulist + (bg * p.n_tiles + tile) * p.t_cap;
  const int ucnt = p.ucnt[bg * p.n_tiles + tile];
  const int last_pos = min(pos0 + P, p.S) - 1;
  const int diag_last = p.causal ? last_pos : min((t + 1) * p.block, p.S) - 1;
  const int n_diag = (diag_last - t * p.block) / kKV + 1;
  const int n_sub = ucnt * spb + n_diag;

  auto sub_tok0 = [&](int s) -> int {
    if (s < ucnt * spb) return ulist[s / spb] * p.block + (s % spb) * kKV;
    return t * p.block + (s - ucnt * spb) * kKV;
  };
  auto load_kv = [&](int s, int buf) {
    const int tok0 = sub_tok0(s);
    T* kd = Ks + buf * kKV * D;
    T* vd = Vs + buf * kKV * D;
    for (int i = tid; i < kKV * NCH; i += NW * 32) {
      const int r = i / NCH, c = i % NCH;
      const int tok = tok0 + r;
      const bool ok = tok < p.S;
      const int64_t off = (int64_t)(ok ? tok : 0) * p.k.ss + c * 8;
      cp_async16(kd + swz<D>(r, c), kg + off, ok);
      const int64_t offv = (int64_t)(ok ? tok : 0) * p.v.ss + c * 8;
      cp_async16(vd + swz<D>(r, c), vg + offv, ok);
    }
    cp_async_commit();
  };
  load_kv(0, 0);

  // ---- per-thread rows
  const int r0 = warp * 16 + (lane >> 2);
  int rpos[2], rhead[2];
  bool rvalid[2];
  RowList lists[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = r0 + 8 * i;
    rpos[i] = pos0 + r / G;
    rhead[i] = g * G + r % G;
    rvalid[i] = (r / G < P) && rpos[i] < p.S;
    const int64_t row = bg * p.S + (rvalid[i] ? rpos[i] : 0);
    const int n = rvalid[i] ? min(max(p.cnt[row], 0), (int)p.t_cap) : 0;
    lists[i].init(p.idx + row * p.t_cap, p.logp + row * p.t_cap, n);
  }
  const float beta = N > 0 ? logf(1.0f / (float)N) : 0.0f;
  const float qk_scale = rsqrtf((float)D) * kLog2e;

  cp_async_wait<1>();
  __syncthreads();
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int r = warp * 16 + (lane & 15);
    const int c = ks * 2 + (lane >> 4);
    ldsm_x4(qa[ks], Qs + swz<D>(r, c));
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m[2] = {kNegInf, kNegInf}, l[2] = {0.f, 0.f};
  float bias[2] = {kNegInf, kNegInf};

  for (int s = 0; s < n_sub; ++s) {
    if (s + 1 < n_sub) {
      load_kv(s + 1, (s + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int buf = s & 1;
    const T* kb = Ks + buf * kKV * D;
    const T* vb = Vs + buf * kKV * D;
    const bool diag = s >= ucnt * spb;
    const int tok0 = sub_tok0(s);
    if (!diag && (s % spb) == 0) {
      const int c = ulist[s / spb];
#pragma unroll
      for (int i = 0; i < 2; ++i) bias[i] = lists[i].bias_for(c);
    } else if (diag) {
      bias[0] = bias[1] = beta;
    }
    const bool active = (rvalid[0] && bias[0] != kNegInf) || (rvalid[1] && bias[1] != kNegInf);
    if (__any_sync(0xffffffffu, active)) {
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t kb4[4];
          const int tok = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int c = ks * 2 + ((lane >> 3) & 1);
          ldsm_x4(kb4, kb + swz<D>(tok, c));
          mma16816<T>(sc[2 * np], qa[ks], kb4[0], kb4[1]);
          mma16816<T>(sc[2 * np + 1], qa[ks], kb4[2], kb4[3]);
        }
      }
      // logits (log2 domain) with bias and masks
      float mx[2] = {kNegInf, kNegInf};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = e >> 1;
          const int tok = tok0 + nt * 8 + 2 * (lane & 3) + (e & 1);
          float x = sc[nt][e] * qk_scale + bias[i] * kLog2e;
          const bool masked = !rvalid[i] || tok >= p.S || (diag && p.causal && tok > rpos[i]) ||
                              bias[i] == kNegInf;
          x = masked ? kNegInf : x;
          sc[nt][e] = x;
          mx[i] = fmaxf(mx[i], x);
        }
      }
      float scale_o[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        const float mn = fmaxf(m[i], mx[i]);
        const float mu = mn == kNegInf ? 0.f : mn;
        scale_o[i] = exp2f(m[i] - mu);
        m[i] = mn;
        l[i] *= scale_o[i];
        mx[i] = mu;
      }
      uint32_t pa[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(sc[nt][0] - mx[0]), p1 = exp2f(sc[nt][1] - mx[0]);
        const float p2 = exp2f(sc[nt][2] - mx[1]), p3 = exp2f(sc[nt][3] - mx[1]);
        l[0] += p0 + p1;
        l[1] += p2 + p3;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][2 * hi] = pack2<T>(p0, p1);
        pa[kk][2 * hi + 1] = pack2<T>(p2, p3);
      }
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        o[dt][0] *= scale_o[0];
        o[dt][1] *= scale_o[0];
        o[dt][2] *= scale_o[1];
        o[dt][3] *= scale_o[1];
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t vb4[4];
          const int tok = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int c = dp * 2 + (lane >> 4);
          ldsm_x4_t(vb4, vb + swz<D>(tok, c));
          mma16816<T>(o[2 * dp], pa[kk], vb4[0], vb4[1]);
          mma16816<T>(o[2 * dp + 1], pa[kk], vb4[2], vb4[3]);
        }
      }
    }
    __syncthreads();
  }

  // ---- epilogue
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
  }
  T* og = static_cast<T*>(const_cast<void*>(p.out.data)) + (int64_t)b * p.out.sb;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!rvalid[i]) continue;
    const float inv = l[i] > 0.f ? 1.0f / l[i] : 0.f;
    T* dst = og + (int64_t)rpos[i] * p.out.ss + (int64_t)rhead[i] * p.out.sh;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      const int col = dt * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(dst + col) = pack2<T>(o[dt][2 * i] * inv, o[dt][2 * i + 1] * inv);
    }
  }
}

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
  const float beta = N > 0 ? logf(1.0f / (float)N) : 0.0f;
  for (int it = 0; it <= n; ++it) {
    const bool diag = it == n;
    const int c = diag ? t : idx[it];
    if (!diag && (c < 0 || c == t || (p.causal ? c >= t : c >= T_))) {
      raise_status(p.status, 1 /* DASH_ERR_INVALID_ARGUMENT */, 201);
      continue;
    }
    const float bias = diag ? beta : logp[it];
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

template <typename T, int D, int NW>
cudaError_t launch_mma(const SparseParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)(16 * NW * D + 4 * kKV * D) * sizeof(T);
  auto kern = sparse_prefill_mma_kernel<T, D, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_tiles, p.Hkv, p.B);
  kern<<<grid, NW * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_mma_rows(const SparseParams& p, cudaStream_t stream) {
  const int rows = p.tile_pos * p.G;
  if (rows == 128) return launch_mma<T, D, 8>(p, stream);
  if (rows == 64) return launch_mma<T, D, 4>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

int sparse_tile_positions(int G, int block) {
  const int p = 128 / G;
  return p < block ? p : block;
}

cudaError_t launch_sparse_prefill(const SparseParams& p, cudaStream_t stream) {
  if (p.dtype == 0) {
    dim3 grid((unsigned)(((int64_t)p.S * p.H + 7) / 8), p.B);
    if (p.D == 128)
      sparse_simt_kernel<128><<<grid, 256, 0, stream>>>(p);
    else
      sparse_simt_kernel<64><<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
  }
  if (p.D == 128) {
    if (p.dtype == 1) return launch_mma_rows<__half, 128>(p, stream);
    return launch_mma_rows<__nv_bfloat16, 128>(p, stream);
  }
  if (p.dtype == 1) return launch_mma_rows<__half, 64>(p, stream);
  return launch_mma_rows<__nv_bfloat16, 64>(p, stream);
}

}  // namespace dash
