// C ABI of libdashattn: argument checks, workspace carving and launches.
// Every entry point validates on the host before launching anything and
// allocates no memory; work goes to the caller's stream.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/dashattn.h"
#include "common.cuh"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

dash_status_t fail(dash_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
dash_status_t fail(dash_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dash_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(DASH_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

dash_status_t ok() {
  g_last_error.clear();
  return DASH_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elt_size(int dtype) { return dtype == DASH_F32 ? 4 : 2; }

// Checks one tensor descriptor.  `name` is used in messages.
dash_status_t check_tensor(const dash_tensor_t* t, const char* name) {
  if (!t) return fail(DASH_ERR_INVALID_ARGUMENT, "%s: null descriptor", name);
  if (!t->data) return fail(DASH_ERR_INVALID_ARGUMENT, "%s: null data pointer", name);
  if (t->dtype != DASH_F32 && t->dtype != DASH_F16 && t->dtype != DASH_BF16)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, t->dtype);
  if (t->b <= 0 || t->s <= 0 || t->h <= 0 || t->d <= 0)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s: extents must be positive (b=%lld s=%lld h=%lld d=%lld)", name,
                (long long)t->b, (long long)t->s, (long long)t->h, (long long)t->d);
  if (t->d != 64 && t->d != 128) return fail(DASH_ERR_UNSUPPORTED, "%s: head dim %lld not in {64, 128}", name, (long long)t->d);
  if (t->s > (1LL << 30) || t->b > 65535 || t->h > 65535)
    return fail(DASH_ERR_UNSUPPORTED, "%s: extents too large", name);
  const int es = elt_size(t->dtype);
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s: data pointer not 16-byte aligned", name);
  if ((t->stride_b * es) % 16 || (t->stride_s * es) % 16 || (t->stride_h * es) % 16)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s: strides must be multiples of 16 bytes", name);
  if (t->stride_b < 0 || t->stride_s < 0 || t->stride_h < 0)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s: negative strides are not supported", name);
  return DASH_OK;
}

dash_status_t check_common(float alpha, int block) {
  if (!(alpha > 1.0f && alpha <= 2.0f)) return fail(DASH_ERR_INVALID_ARGUMENT, "alpha %g not in (1, 2]", alpha);
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  return DASH_OK;
}

dash_status_t check_group(int64_t H, int64_t Hkv) {
  if (Hkv <= 0 || H % Hkv) return fail(DASH_ERR_INVALID_ARGUMENT, "heads %lld not a multiple of kv heads %lld", (long long)H, (long long)Hkv);
  const int64_t G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(DASH_ERR_UNSUPPORTED, "group size %lld not in {1, 2, 4, 8}", (long long)G);
  return DASH_OK;
}

dash::View view(const dash_tensor_t* t) { return dash::View{t->data, t->stride_b, t->stride_s, t->stride_h}; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Workspace of dash_attn_fwd.
struct FwdLayout {
  size_t status, summ, split, wide, idx, logp, cnt, ulist, umask, ucnt, usteps, plist, pmask, pcnt, psteps, total;
  int64_t T, n_tiles, n_pairs;
  int tile_pos, n_slots;
};

// Scratch slots of the segmented routing kernel (tiles with more than 512
// candidate columns): one per SM (one of its CTAs fills an SM) and 32 spare,
// so that a CTA never waits for the release of the CTA it replaces; none when
// no tile can be that wide.
int wide_slots(int64_t t_cap) { return t_cap > dash::route_tc_max_cols() ? num_sms() + 32 : 0; }
size_t wide_bytes(int64_t t_cap) {
  const int n = wide_slots(t_cap);
  return n ? dash::route_wide_scratch_bytes(t_cap, n) : 0;
}

FwdLayout fwd_layout(int64_t B, int64_t S, int64_t H, int64_t Hkv, int64_t D, int block) {
  FwdLayout L{};
  const int64_t G = H / Hkv;
  L.T = (S + block - 1) / block;
  L.tile_pos = dash::sparse_tile_positions((int)G, block);
  L.n_tiles = (S + L.tile_pos - 1) / L.tile_pos;
  size_t off = 0;
  L.status = off;
  off = align256(off + sizeof(dash::DeviceStatus));
  L.summ = off;
  off = align256(off + (size_t)B * Hkv * L.T * D * 4);
  L.split = off;  // summaries split for the tensor-core routing kernel
  off = align256(off + dash::route_split_bytes(B, Hkv, L.T, (int)D));
  L.wide = off;  // scratch slots of the segmented routing kernel
  L.n_slots = wide_slots(L.T);
  off = align256(off + wide_bytes(L.T));
  L.idx = off;
  off = align256(off + (size_t)B * Hkv * S * L.T * 4);
  L.logp = off;
  off = align256(off + (size_t)B * Hkv * S * L.T * 4);
  L.cnt = off;
  off = align256(off + (size_t)B * Hkv * S * 4);
  L.ulist = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * L.T * 4);
  L.umask = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * L.T * 16);
  L.ucnt = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * 4);
  L.usteps = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * 4);
  L.n_pairs = (L.n_tiles + 1) / 2;
  L.plist = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * L.T * 4);
  L.pmask = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * L.T * 32);
  L.pcnt = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * 4);
  L.psteps = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * 4);
  L.total = off;
  return L;
}

struct SparseLayout {
  size_t status, ulist, umask, ucnt, usteps, plist, pmask, pcnt, psteps, total;
  int64_t n_tiles, n_pairs;
  int tile_pos;
};

SparseLayout sparse_layout(int64_t B, int64_t S, int64_t H, int64_t Hkv, int block, int64_t t_cap) {
  SparseLayout L{};
  L.tile_pos = dash::sparse_tile_positions((int)(H / Hkv), block);
  L.n_tiles = (S + L.tile_pos - 1) / L.tile_pos;
  size_t off = 0;
  L.status = off;
  off = align256(off + sizeof(dash::DeviceStatus));
  L.ulist = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * t_cap * 4);
  L.umask = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * t_cap * 16);
  L.ucnt = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * 4);
  L.usteps = off;
  off = align256(off + (size_t)B * Hkv * L.n_tiles * 4);
  L.n_pairs = (L.n_tiles + 1) / 2;
  L.plist = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * t_cap * 4);
  L.pmask = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * t_cap * 32);
  L.pcnt = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * 4);
  L.psteps = off;
  off = align256(off + (size_t)B * Hkv * L.n_pairs * 4);
  L.total = off;
  return L;
}

struct DecodeLayout {
  size_t status, scores, idx, logp, cnt, items, n_items, pair_base, part_o, part_ml, total;
  int64_t max_items;
  int chunk;
};

DecodeLayout decode_layout(int64_t B, int64_t H, int64_t Hkv, int64_t D, int block, int64_t t_cap) {
  DecodeLayout L{};
  const int64_t G = H / Hkv;
  L.chunk = block == 64 ? 16 : 8;
  L.max_items = dash::decode_max_items(B, Hkv, t_cap, L.chunk);
  size_t off = 0;
  L.status = off;
  off = align256(off + sizeof(dash::DeviceStatus));
  L.scores = off;
  off = align256(off + (size_t)B * Hkv * G * t_cap * 4);
  L.idx = off;
  off = align256(off + (size_t)B * Hkv * t_cap * 4);
  L.logp = off;
  off = align256(off + (size_t)B * Hkv * t_cap * 4);
  L.cnt = off;
  off = align256(off + (size_t)B * Hkv * 4);
  L.items = off;
  off = align256(off + (size_t)L.max_items * 2 * 4);
  L.n_items = off;
  off = align256(off + 4);
  L.pair_base = off;
  off = align256(off + (size_t)B * Hkv * 4);
  L.part_o = off;
  off = align256(off + (size_t)L.max_items * G * D * 4);
  L.part_ml = off;
  off = align256(off + (size_t)L.max_items * G * 2 * 4);
  L.total = off;
  return L;
}

// Workspace of dash_attn_bwd.
struct BwdLayout {
  size_t status, summ, split, wide, idx, logp, cnt, tau, lse, dd, dz, umask, kbar, ds, lists, rmask, rrank, tbits,
      total;
  int64_t T, n_words;
  int n_slots;
  SparseLayout sl;  // tile work lists of the stage-2 pass that takes each row's log-sum-exp
};

BwdLayout bwd_layout(int64_t B, int64_t S, int64_t H, int64_t Hkv, int64_t D, int block) {
  BwdLayout L{};
  const int64_t G = H / Hkv;
  L.T = (S + block - 1) / block;
  L.n_words = (L.T + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t& field, size_t bytes) {
    field = off;
    off = align256(off + bytes);
  };
  take(L.status, sizeof(dash::DeviceStatus));
  take(L.summ, (size_t)B * Hkv * L.T * D * 4);
  take(L.split, dash::route_split_bytes(B, Hkv, L.T, (int)D));
  L.n_slots = wide_slots(L.T);
  take(L.wide, wide_bytes(L.T));
  take(L.idx, (size_t)B * Hkv * S * L.T * 4);
  take(L.logp, (size_t)B * Hkv * S * L.T * 4);
  take(L.cnt, (size_t)B * Hkv * S * 4);
  take(L.tau, (size_t)B * H * S * 4);
  take(L.lse, (size_t)B * H * S * 4);
  take(L.dd, (size_t)B * H * S * 4);
  take(L.dz, (size_t)B * Hkv * S * L.T * G * 4);
  take(L.umask, (size_t)B * Hkv * L.T * L.n_words * 4);
  take(L.kbar, (size_t)B * Hkv * L.T * D * 4);
  take(L.ds, (size_t)B * Hkv * L.T * D * 4);
  L.sl = sparse_layout(B, S, H, Hkv, block, L.T);
  take(L.lists, L.sl.total);
  take(L.rmask, (size_t)B * Hkv * S * L.n_words * 4);
  take(L.rrank, (size_t)B * Hkv * S * L.n_words * 4);
  take(L.tbits, (size_t)B * Hkv * L.sl.n_tiles * L.n_words * 4);
  L.total = off;
  return L;
}

template <typename P>
P* at(void* base, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(base) + off);
}

dash_status_t check_fwd_shapes(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                               const dash_tensor_t* out) {
  dash_status_t st;
  if ((st = check_tensor(q, "q")) || (st = check_tensor(k, "k")) || (st = check_tensor(v, "v")) ||
      (st = check_tensor(out, "out")))
    return st;
  if (q->dtype != k->dtype || q->dtype != v->dtype || q->dtype != out->dtype)
    return fail(DASH_ERR_INVALID_ARGUMENT, "q, k, v and out must share one dtype");
  if (k->b != q->b || v->b != q->b || out->b != q->b) return fail(DASH_ERR_INVALID_ARGUMENT, "batch mismatch");
  if (k->d != q->d || v->d != q->d || out->d != q->d) return fail(DASH_ERR_INVALID_ARGUMENT, "head dim mismatch");
  if (k->h != v->h) return fail(DASH_ERR_INVALID_ARGUMENT, "k and v head counts differ");
  if (out->h != q->h || out->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "out must have q's shape");
  return check_group(q->h, k->h);
}

}  // namespace

namespace dash {
dash_status_t set_last_error(dash_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}
}  // namespace dash

extern "C" {

int dash_attn_version(void) { return 100; }

const char* dash_attn_last_error(void) { return g_last_error.c_str(); }

size_t dash_attn_fwd_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block) {
  if (check_tensor(q, "q") || check_tensor(k, "k") || (block != 64 && block != 128) || check_group(q->h, k->h))
    return 0;
  return fwd_layout(q->b, q->s, q->h, k->h, q->d, block).total;
}

dash_status_t dash_attn_fwd_workspace_lists(const dash_tensor_t* q, const dash_tensor_t* k, int block,
                                            size_t* summ_offset, size_t* idx_offset, size_t* logp_offset,
                                            size_t* cnt_offset) {
  dash_status_t st;
  if ((st = check_tensor(q, "q")) || (st = check_tensor(k, "k")) || (st = check_group(q->h, k->h))) return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  const FwdLayout L = fwd_layout(q->b, q->s, q->h, k->h, q->d, block);
  if (summ_offset) *summ_offset = L.summ;
  if (idx_offset) *idx_offset = L.idx;
  if (logp_offset) *logp_offset = L.logp;
  if (cnt_offset) *cnt_offset = L.cnt;
  return ok();
}

dash_status_t dash_attn_summarize(const dash_tensor_t* k, const int32_t* seqlens, const float* w_s, int block,
                                  float* summaries, int64_t t_cap, int64_t first_block, dash_stream_t stream) {
  return dash_attn_summarize_sdpa(k, seqlens, w_s, nullptr, block, summaries, t_cap, first_block, stream);
}

dash_status_t dash_attn_summarize_sdpa(const dash_tensor_t* k, const int32_t* seqlens, const float* w_s,
                                       const float* qbar, int block, float* summaries, int64_t t_cap,
                                       int64_t first_block, dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_tensor(k, "k"))) return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (!w_s || !summaries) return fail(DASH_ERR_INVALID_ARGUMENT, "null w_s or summaries");
  if (reinterpret_cast<uintptr_t>(summaries) % 16) return fail(DASH_ERR_INVALID_ARGUMENT, "summaries not 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(w_s) % 16 || reinterpret_cast<uintptr_t>(qbar) % 16)
    return fail(DASH_ERR_INVALID_ARGUMENT, "w_s or qbar not 16-byte aligned");
  const int64_t T = (k->s + block - 1) / block;
  if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(S / block) = %lld", (long long)t_cap, (long long)T);
  if (first_block < 0) return fail(DASH_ERR_INVALID_ARGUMENT, "first_block < 0");
  dash::PoolParams p{};
  p.k = view(k);
  p.dtype = k->dtype;
  p.B = (int)k->b;
  p.S = (int)k->s;
  p.Hkv = (int)k->h;
  p.D = (int)k->d;
  p.block = block;
  p.seqlens = seqlens;
  p.w_s = w_s;
  p.qbar = qbar;
  p.summaries = summaries;
  p.t_cap = t_cap;
  p.first_block = first_block;
  cudaError_t e = dash::launch_pool(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "summarize");
  return ok();
}

}  // extern "C"

namespace {

struct TileLists {
  int32_t* ulist;
  uint4* umask;
  int32_t* ucnt;
  int32_t* usteps;
  int32_t* plist;
  uint4* pmask;
  int32_t* pcnt;
  int32_t* psteps;
  int64_t n_pairs;
};

// Prefill routing.  f16/bf16 tiles whose logit row fits in TMEM run on the
// tensor cores (and, when `tl` is given, also write the stage-2 work lists of
// their tiles); the remaining positions, and fp32 inputs, run on the CUDA
// cores.  Returns in *first_cuda_tile the first tile routed on the CUDA
// cores (whose work lists still have to be built).
dash_status_t run_route(const dash_tensor_t* q, const float* summaries, int64_t kv_heads, int64_t t_cap, float alpha,
                        int block, int causal, int32_t* idx, float* logp, int32_t* cnt, float* tau, float* p_dense,
                        const TileLists* tl, dash::DeviceStatus* status, cudaStream_t stream, int* first_cuda_tile,
                        float* split_buf = nullptr, void* wide_buf = nullptr) {
  const int G = (int)(q->h / kv_heads);
  dash::RouteParams p{};
  p.q = view(q);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.S = (int)q->s;
  p.H = (int)q->h;
  p.Hkv = (int)kv_heads;
  p.G = G;
  p.D = (int)q->d;
  p.block = block;
  p.causal = causal ? 1 : 0;
  p.alpha = alpha;
  p.summaries = summaries;
  p.t_cap = t_cap;
  p.idx = idx;
  p.logp = logp;
  p.cnt = cnt;
  p.tau = tau;
  p.p_dense = p_dense;
  p.status = status;
  const int P = dash::sparse_tile_positions(G, block);
  const int n_tiles = (int)((q->s + P - 1) / P);
  const int n_blocks = (int)((q->s + block - 1) / block);
  int split = 0;
  if (q->dtype != DASH_F32) {
    // tiles [0, narrow) fit TMEM; the rest run the segmented kernel when its
    // scratch (and the split summaries it streams) are given, else CUDA cores
    const int max_cols = dash::route_tc_max_cols();
    int narrow;
    if (causal) {
      narrow = (int)(((int64_t)(max_cols + 1) * block) / P);
      if (narrow > n_tiles) narrow = n_tiles;
    } else {
      narrow = n_blocks <= max_cols ? n_tiles : 0;
    }
    const bool wide = wide_buf && split_buf && narrow < n_tiles && n_blocks <= dash::route_tc_wide_max_cols();
    dash::TileOut to{};
    if (tl) to = dash::TileOut{tl->ulist, tl->umask, tl->ucnt, tl->usteps, n_tiles};
    if (split_buf && (narrow > 0 || wide)) {
      cudaError_t e = dash::launch_route_split(p, split_buf, stream);
      if (e != cudaSuccess) return cuda_fail(e, "route (split summaries)");
      p.summ_split = split_buf;
    }
    cudaError_t e = dash::launch_route_prefill_tc(p, to, 0, narrow, stream);
    if (e != cudaSuccess) return cuda_fail(e, "route (tensor cores)");
    split = narrow;
    if (wide) {
      const int n_slots = wide_slots(t_cap);
      const dash::WideScratch w = dash::route_wide_scratch(wide_buf, t_cap, n_slots);
      e = cudaMemsetAsync(w.locks, 0, (size_t)n_slots * 4, stream);
      if (e != cudaSuccess) return cuda_fail(e, "memset");
      e = dash::launch_route_prefill_tc_wide(p, to, narrow, n_tiles - narrow, w, stream);
      if (e != cudaSuccess) return cuda_fail(e, "route (tensor cores, segmented)");
      split = n_tiles;
    }
    p.summ_split = nullptr;
  }
  p.pos_begin = split * P;
  if (p.pos_begin < p.S) {
    cudaError_t e = dash::launch_route_prefill(p, stream);
    if (e != cudaSuccess) return cuda_fail(e, "route");
  }
  if (first_cuda_tile) *first_cuda_tile = split;
  return DASH_OK;
}

}  // namespace

extern "C" {

size_t dash_attn_route_workspace_size(const dash_tensor_t* q, int64_t kv_heads, int64_t t_cap, int decode) {
  if (check_tensor(q, "q") || check_group(q->h, kv_heads) || t_cap <= 0) return 0;
  if (!decode)  // optional in prefill mode: split summaries, then the segmented kernel's scratch
    return align256(dash::route_split_bytes(q->b, kv_heads, t_cap, (int)q->d)) + wide_bytes(t_cap);
  return decode_layout(q->b, q->h, kv_heads, q->d, 64, t_cap).idx;  // status + per-head logits
}

dash_status_t dash_attn_route(const dash_tensor_t* q, const float* summaries, int64_t kv_heads, int64_t t_cap,
                              const int32_t* seqlens, float alpha, int block, int causal, int32_t* idx, float* logp,
                              int32_t* cnt, float* tau, float* p_dense, void* workspace, size_t workspace_bytes,
                              dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_tensor(q, "q")) || (st = check_common(alpha, block)) || (st = check_group(q->h, kv_heads))) return st;
  if (!summaries || !idx || !logp || !cnt) return fail(DASH_ERR_INVALID_ARGUMENT, "null summaries/idx/logp/cnt");
  if (reinterpret_cast<uintptr_t>(summaries) % 16) return fail(DASH_ERR_INVALID_ARGUMENT, "summaries not 16-byte aligned");
  const int G = (int)(q->h / kv_heads);
  if (!seqlens) {
    const int64_t T = (q->s + block - 1) / block;
    if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(S / block)", (long long)t_cap);
    if (T > 4096) return fail(DASH_ERR_UNSUPPORTED, "more than 4096 blocks per sequence");
    // a workspace, when given, holds the split summaries of the tensor-core kernel
    float* split = nullptr;
    void* wide = nullptr;
    const size_t split_bytes = align256(dash::route_split_bytes(q->b, kv_heads, t_cap, (int)q->d));
    if (workspace && reinterpret_cast<uintptr_t>(workspace) % 256 == 0 && workspace_bytes >= split_bytes) {
      split = static_cast<float*>(workspace);
      if (wide_bytes(t_cap) && workspace_bytes >= split_bytes + wide_bytes(t_cap))
        wide = static_cast<char*>(workspace) + split_bytes;
    }
    st = run_route(q, summaries, kv_heads, t_cap, alpha, block, causal, idx, logp, cnt, tau, p_dense, nullptr,
                   nullptr, (cudaStream_t)stream, nullptr, split, wide);
    return st ? st : ok();
  }
  if (q->s != 1) return fail(DASH_ERR_INVALID_ARGUMENT, "decode-mode route needs q with s == 1");
  if (!causal) return fail(DASH_ERR_UNSUPPORTED, "decode-mode route is causal");
  if (t_cap > 4096) return fail(DASH_ERR_UNSUPPORTED, "t_cap above 4096");
  const DecodeLayout L = decode_layout(q->b, q->h, kv_heads, q->d, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "decode-mode route needs a 256-byte aligned workspace");
  if (workspace_bytes < L.idx)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.idx);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  dash::DecodeParams p{};
  p.sigma = 1.0f;
  p.c_lo = 0;
  p.c_hi = (int)t_cap;
  p.summ_cap = t_cap;
  p.q = view(q);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.Lmax = (int)(t_cap * block);
  p.H = (int)q->h;
  p.Hkv = (int)kv_heads;
  p.G = G;
  p.D = (int)q->d;
  p.block = block;
  p.alpha = alpha;
  p.seqlens = seqlens;
  p.summaries = summaries;
  p.t_cap = t_cap;
  p.scores = at<float>(workspace, L.scores);
  p.idx = idx;
  p.logp = logp;
  p.cnt = cnt;
  p.tau = tau;
  p.p_dense = p_dense;
  p.status = at<dash::DeviceStatus>(workspace, L.status);
  e = dash::launch_decode_route(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode route");
  return ok();
}

size_t dash_attn_sparse_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block, int64_t t_cap) {
  if (check_tensor(q, "q") || check_tensor(k, "k") || (block != 64 && block != 128) || check_group(q->h, k->h))
    return 0;
  return sparse_layout(q->b, q->s, q->h, k->h, block, t_cap).total;
}

static dash_status_t run_sparse(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                int causal, float sigma, dash_tensor_t* out, const TileLists& tl, int tile_pos,
                                int64_t n_tiles, int union_tile0, dash::DeviceStatus* status,
                                cudaStream_t stream, const uint32_t* mask = nullptr, int n_words = 0,
                                const float* logp_dense = nullptr, long long wait_cycles = 0,
                                int stall_producer = 0, float* lse = nullptr, int skip_out = 0) {
  if (q->dtype != DASH_F32 && union_tile0 < n_tiles) {
    dash::UnionParams u{};
    u.B = (int)q->b;
    u.S = (int)q->s;
    u.Hkv = (int)k->h;
    u.block = block;
    u.tile_pos = tile_pos;
    u.n_tiles = (int)n_tiles;
    u.tile0 = union_tile0;
    u.t_cap = t_cap;
    u.idx = idx;
    u.cnt = cnt;
    u.ulist = tl.ulist;
    u.umask = tl.umask;
    u.ucnt = tl.ucnt;
    u.usteps = tl.usteps;
    u.causal = causal ? 1 : 0;
    u.status = status;
    u.mask = mask;
    u.n_words = n_words;
    cudaError_t e = dash::launch_union(u, stream);
    if (e != cudaSuccess) return cuda_fail(e, "union");
  }
  if (q->dtype != DASH_F32) {
    dash::PairParams pp{};
    pp.B = (int)q->b;
    pp.S = (int)q->s;
    pp.Hkv = (int)k->h;
    pp.block = block;
    pp.tile_pos = tile_pos;
    pp.n_tiles = (int)n_tiles;
    pp.n_pairs = (int)tl.n_pairs;
    pp.causal = causal ? 1 : 0;
    pp.t_cap = t_cap;
    pp.ulist = tl.ulist;
    pp.umask = tl.umask;
    pp.ucnt = tl.ucnt;
    pp.plist = tl.plist;
    pp.pmask = tl.pmask;
    pp.pcnt = tl.pcnt;
    pp.psteps = tl.psteps;
    cudaError_t e = dash::launch_pairs(pp, stream);
    if (e != cudaSuccess) return cuda_fail(e, "pair lists");
  }
  dash::SparseParams p{};
  p.q = view(q);
  p.k = view(k);
  p.v = view(v);
  p.out = view(out);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.S = (int)q->s;
  p.H = (int)q->h;
  p.Hkv = (int)k->h;
  p.G = (int)(q->h / k->h);
  p.D = (int)q->d;
  p.block = block;
  p.causal = causal ? 1 : 0;
  p.t_cap = t_cap;
  p.idx = idx;
  p.logp = logp;
  p.cnt = cnt;
  p.plist = tl.plist;
  p.pmask = tl.pmask;
  p.pcnt = tl.pcnt;
  p.psteps = tl.psteps;
  p.n_pairs = (int)tl.n_pairs;
  p.tile_pos = tile_pos;
  p.n_tiles = (int)n_tiles;
  p.sigma = sigma;
  p.status = status;
  p.logp_dense = logp_dense;
  p.wait_cycles = wait_cycles;
  p.stall_producer = stall_producer;
  p.lse = lse;
  p.skip_out = skip_out;
  cudaError_t e = dash::launch_sparse_prefill(p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sparse attention");
  return DASH_OK;
}

static dash_status_t read_options(const dash_options_t* opts, bool qbar_allowed, float* sigma, const float** qbar) {
  *sigma = 1.0f;
  *qbar = nullptr;
  if (!opts) return DASH_OK;
  if (!(opts->sigma >= 0.0f) || opts->sigma > 3.0e38f)
    return fail(DASH_ERR_INVALID_ARGUMENT, "sigma must be finite and >= 0");
  if (opts->qbar && !qbar_allowed) return fail(DASH_ERR_INVALID_ARGUMENT, "qbar is not used here; pass NULL");
  *sigma = opts->sigma;
  *qbar = opts->qbar;
  return DASH_OK;
}

dash_status_t dash_attn_sparse(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                               const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                               int causal, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                               dash_stream_t stream) {
  return dash_attn_sparse_ex(q, k, v, idx, logp, cnt, t_cap, block, causal, out, workspace, workspace_bytes, nullptr,
                             stream);
}

dash_status_t dash_attn_sparse_ex(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                  const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                  int causal, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                  const dash_options_t* opts, dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if ((st = check_fwd_shapes(q, k, v, out))) return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (k->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "prefill needs k and q of equal length");
  if (!idx || !logp || !cnt) return fail(DASH_ERR_INVALID_ARGUMENT, "null routing lists");
  const int64_t T = (q->s + block - 1) / block;
  if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(S / block)", (long long)t_cap);
  const SparseLayout L = sparse_layout(q->b, q->s, q->h, k->h, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  const TileLists tl{at<int32_t>(workspace, L.ulist), at<uint4>(workspace, L.umask), at<int32_t>(workspace, L.ucnt),
                     at<int32_t>(workspace, L.usteps), at<int32_t>(workspace, L.plist), at<uint4>(workspace, L.pmask),
                     at<int32_t>(workspace, L.pcnt), at<int32_t>(workspace, L.psteps), L.n_pairs};
  st = run_sparse(q, k, v, idx, logp, cnt, t_cap, block, causal, sigma, out, tl, L.tile_pos, L.n_tiles, 0,
                  at<dash::DeviceStatus>(workspace, L.status), s);
  return st ? st : ok();
}

dash_status_t dash_attn_debug_sparse_stalled(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                             const int32_t* idx, const float* logp, const int32_t* cnt, int64_t t_cap,
                                             int block, int causal, dash_tensor_t* out, void* workspace,
                                             size_t workspace_bytes, int64_t wait_cycles, dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_fwd_shapes(q, k, v, out))) return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "the stalled stage 2 is the f16/bf16 kernel");
  if (k->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "prefill needs k and q of equal length");
  if (!idx || !logp || !cnt) return fail(DASH_ERR_INVALID_ARGUMENT, "null routing lists");
  if (wait_cycles < 1024 || wait_cycles > (1ll << 31))
    return fail(DASH_ERR_INVALID_ARGUMENT, "wait_cycles must be in [1024, 2^31]");
  const int64_t T = (q->s + block - 1) / block;
  if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(S / block)", (long long)t_cap);
  const SparseLayout L = sparse_layout(q->b, q->s, q->h, k->h, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  const TileLists tl{at<int32_t>(workspace, L.ulist), at<uint4>(workspace, L.umask), at<int32_t>(workspace, L.ucnt),
                     at<int32_t>(workspace, L.usteps), at<int32_t>(workspace, L.plist), at<uint4>(workspace, L.pmask),
                     at<int32_t>(workspace, L.pcnt), at<int32_t>(workspace, L.psteps), L.n_pairs};
  st = run_sparse(q, k, v, idx, logp, cnt, t_cap, block, causal, 1.0f, out, tl, L.tile_pos, L.n_tiles, 0,
                  at<dash::DeviceStatus>(workspace, L.status), s, nullptr, 0, nullptr, wait_cycles, 1);
  return st ? st : ok();
}

dash_status_t dash_attn_sparse_mask(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                                    const uint32_t* mask, int64_t n_words, const float* logp, int64_t t_cap, int block,
                                    int causal, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                    const dash_options_t* opts, dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if ((st = check_fwd_shapes(q, k, v, out))) return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "the mask form takes f16 or bf16 inputs");
  if (k->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "prefill needs k and q of equal length");
  if (!mask || !logp) return fail(DASH_ERR_INVALID_ARGUMENT, "null mask or logp");
  if (reinterpret_cast<uintptr_t>(mask) % 4 || reinterpret_cast<uintptr_t>(logp) % 4)
    return fail(DASH_ERR_INVALID_ARGUMENT, "mask and logp must be 4-byte aligned");
  const int64_t T = (q->s + block - 1) / block;
  if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(S / block)", (long long)t_cap);
  if (T > 4096) return fail(DASH_ERR_UNSUPPORTED, "more than 4096 blocks per sequence");
  if (n_words * 32 < T || n_words > 128)
    return fail(DASH_ERR_INVALID_ARGUMENT, "n_words %lld must cover ceil(S / block) blocks, at most 128",
                (long long)n_words);
  const SparseLayout L = sparse_layout(q->b, q->s, q->h, k->h, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  const TileLists tl{at<int32_t>(workspace, L.ulist), at<uint4>(workspace, L.umask), at<int32_t>(workspace, L.ucnt),
                     at<int32_t>(workspace, L.usteps), at<int32_t>(workspace, L.plist), at<uint4>(workspace, L.pmask),
                     at<int32_t>(workspace, L.pcnt), at<int32_t>(workspace, L.psteps), L.n_pairs};
  st = run_sparse(q, k, v, nullptr, nullptr, nullptr, t_cap, block, causal, sigma, out, tl, L.tile_pos, L.n_tiles, 0,
                  at<dash::DeviceStatus>(workspace, L.status), s, mask, (int)n_words, logp);
  return st ? st : ok();
}

dash_status_t dash_attn_fwd(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v, const float* w_s,
                            float alpha, int block, int causal, dash_tensor_t* out, void* workspace,
                            size_t workspace_bytes, dash_stream_t stream) {
  return dash_attn_fwd_ex(q, k, v, w_s, alpha, block, causal, out, workspace, workspace_bytes, nullptr, stream);
}

dash_status_t dash_attn_fwd_ex(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                               const float* w_s, float alpha, int block, int causal, dash_tensor_t* out,
                               void* workspace, size_t workspace_bytes, const dash_options_t* opts,
                               dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, true, &sigma, &qbar))) return st;
  if ((st = check_fwd_shapes(q, k, v, out)) || (st = check_common(alpha, block))) return st;
  if (k->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "prefill needs k and q of equal length");
  if (!w_s) return fail(DASH_ERR_INVALID_ARGUMENT, "null w_s");
  const FwdLayout L = fwd_layout(q->b, q->s, q->h, k->h, q->d, block);
  if (L.T > 4096) return fail(DASH_ERR_UNSUPPORTED, "more than 4096 blocks per sequence");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  float* summ = at<float>(workspace, L.summ);
  if ((st = dash_attn_summarize_sdpa(k, nullptr, w_s, qbar, block, summ, L.T, 0, stream))) return st;
  int32_t* idx = at<int32_t>(workspace, L.idx);
  float* logp = at<float>(workspace, L.logp);
  int32_t* cnt = at<int32_t>(workspace, L.cnt);
  const TileLists tl{at<int32_t>(workspace, L.ulist), at<uint4>(workspace, L.umask), at<int32_t>(workspace, L.ucnt),
                     at<int32_t>(workspace, L.usteps), at<int32_t>(workspace, L.plist), at<uint4>(workspace, L.pmask),
                     at<int32_t>(workspace, L.pcnt), at<int32_t>(workspace, L.psteps), L.n_pairs};
  dash::DeviceStatus* dst = at<dash::DeviceStatus>(workspace, L.status);
  int first_cuda_tile = 0;
  if ((st = run_route(q, summ, k->h, L.T, alpha, block, causal, idx, logp, cnt, nullptr, nullptr, &tl, dst, s,
                      &first_cuda_tile, at<float>(workspace, L.split), L.n_slots ? at<char>(workspace, L.wide) : nullptr)))
    return st;
  st = run_sparse(q, k, v, idx, logp, cnt, L.T, block, causal, sigma, out, tl, L.tile_pos, L.n_tiles, first_cuda_tile,
                  dst, s);
  return st ? st : ok();
}

size_t dash_attn_bwd_workspace_size(const dash_tensor_t* q, const dash_tensor_t* k, int block) {
  if (check_tensor(q, "q") || check_tensor(k, "k") || (block != 64 && block != 128) || check_group(q->h, k->h))
    return 0;
  return bwd_layout(q->b, q->s, q->h, k->h, q->d, block).total;
}

static dash_status_t check_grad(const dash_tensor_t* g, const dash_tensor_t* like, const char* name) {
  dash_status_t st;
  if ((st = check_tensor(g, name))) return st;
  if (g->dtype != DASH_F32) return fail(DASH_ERR_INVALID_ARGUMENT, "%s must be fp32", name);
  if (g->b != like->b || g->s != like->s || g->h != like->h || g->d != like->d)
    return fail(DASH_ERR_INVALID_ARGUMENT, "%s must have the shape of its input", name);
  return DASH_OK;
}

dash_status_t dash_attn_bwd(const dash_tensor_t* q, const dash_tensor_t* k, const dash_tensor_t* v,
                            const float* w_s, const dash_tensor_t* out, const dash_tensor_t* dout, float alpha,
                            int block, int causal, const dash_options_t* opts, dash_tensor_t* dq, dash_tensor_t* dk,
                            dash_tensor_t* dv, float* dw_s, void* workspace, size_t workspace_bytes,
                            dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if ((st = check_fwd_shapes(q, k, v, out)) || (st = check_common(alpha, block))) return st;
  if ((st = check_tensor(dout, "dout"))) return st;
  if (dout->dtype != q->dtype || dout->b != q->b || dout->s != q->s || dout->h != q->h || dout->d != q->d)
    return fail(DASH_ERR_INVALID_ARGUMENT, "dout must have q's shape and dtype");
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "the backward pass takes f16 or bf16 inputs");
  if (k->s != q->s) return fail(DASH_ERR_INVALID_ARGUMENT, "prefill needs k and q of equal length");
  if ((st = check_grad(dq, q, "dq")) || (st = check_grad(dk, k, "dk")) || (st = check_grad(dv, v, "dv"))) return st;
  if (!w_s || !dw_s) return fail(DASH_ERR_INVALID_ARGUMENT, "null w_s or dw_s");
  if (reinterpret_cast<uintptr_t>(w_s) % 16 || reinterpret_cast<uintptr_t>(dw_s) % 16)
    return fail(DASH_ERR_INVALID_ARGUMENT, "w_s and dw_s must be 16-byte aligned");
  const BwdLayout L = bwd_layout(q->b, q->s, q->h, k->h, q->d, block);
  if (L.T > 4096) return fail(DASH_ERR_UNSUPPORTED, "more than 4096 blocks per sequence");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  float* summ = at<float>(workspace, L.summ);
  if ((st = dash_attn_summarize_sdpa(k, nullptr, w_s, nullptr, block, summ, L.T, 0, stream))) return st;
  dash::DeviceStatus* dst = at<dash::DeviceStatus>(workspace, L.status);
  int32_t* idx = at<int32_t>(workspace, L.idx);
  float* logp = at<float>(workspace, L.logp);
  int32_t* cnt = at<int32_t>(workspace, L.cnt);
  float* tau = at<float>(workspace, L.tau);
  if ((st = run_route(q, summ, k->h, L.T, alpha, block, causal, idx, logp, cnt, tau, nullptr, nullptr, dst, s, nullptr,
                      at<float>(workspace, L.split), L.n_slots ? at<char>(workspace, L.wide) : nullptr)))
    return st;
  // each row's log-sum-exp: the forward's stage-2 kernel on the same lists,
  // without writing an output
  float* lse = at<float>(workspace, L.lse);
  {
    char* lw = at<char>(workspace, L.lists);
    const TileLists tl{at<int32_t>(lw, L.sl.ulist), at<uint4>(lw, L.sl.umask), at<int32_t>(lw, L.sl.ucnt),
                       at<int32_t>(lw, L.sl.usteps), at<int32_t>(lw, L.sl.plist), at<uint4>(lw, L.sl.pmask),
                       at<int32_t>(lw, L.sl.pcnt), at<int32_t>(lw, L.sl.psteps), L.sl.n_pairs};
    dash_tensor_t scratch_out = *out;  // not written (skip_out)
    if ((st = run_sparse(q, k, v, idx, logp, cnt, L.T, block, causal, sigma, &scratch_out, tl, L.sl.tile_pos,
                         L.sl.n_tiles, 0, dst, s, nullptr, 0, nullptr, 0, 0, lse, 1)))
      return st;
    // which tiles hold which blocks, and which blocks each row selected, as bit masks
    e = dash::launch_tile_bits(tl.ulist, tl.ucnt, q->b * k->h * L.sl.n_tiles, L.T, at<uint32_t>(workspace, L.tbits),
                               (int)L.n_words, s);
    if (e != cudaSuccess) return cuda_fail(e, "tile bits");
    e = dash::launch_lists_to_mask(idx, cnt, q->b * k->h * q->s, L.T, at<uint32_t>(workspace, L.rmask),
                                   (int)L.n_words, s);
    if (e != cudaSuccess) return cuda_fail(e, "row masks");
    e = dash::launch_row_ranks(at<uint32_t>(workspace, L.rmask), q->b * k->h * q->s, (int)L.n_words,
                               at<int32_t>(workspace, L.rrank), s);
    if (e != cudaSuccess) return cuda_fail(e, "row ranks");
  }
  dash::BwdParams p{};
  p.idx = idx;
  p.logp = logp;
  p.cnt = cnt;
  p.tau = tau;
  p.q = view(q);
  p.k = view(k);
  p.v = view(v);
  p.o = view(out);
  p.dout = view(dout);
  p.dq = view(dq);
  p.dk = view(dk);
  p.dv = view(dv);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.S = (int)q->s;
  p.H = (int)q->h;
  p.Hkv = (int)k->h;
  p.G = (int)(q->h / k->h);
  p.D = (int)q->d;
  p.block = block;
  p.causal = causal ? 1 : 0;
  p.alpha = alpha;
  p.sigma = sigma;
  p.w_s = w_s;
  p.summaries = summ;
  p.t_cap = L.T;
  p.n_qblocks = (int)L.T;
  p.n_words = (int)L.n_words;
  p.lse = lse;
  p.dd = at<float>(workspace, L.dd);
  p.dz = at<float>(workspace, L.dz);
  p.umask = at<uint32_t>(workspace, L.umask);
  p.kbar = at<float>(workspace, L.kbar);
  p.ds = at<float>(workspace, L.ds);
  p.dw_s = dw_s;
  p.status = dst;
  p.tbits = at<uint32_t>(workspace, L.tbits);
  p.rmask = at<uint32_t>(workspace, L.rmask);
  p.rrank = at<int32_t>(workspace, L.rrank);
  p.n_tiles = (int)L.sl.n_tiles;
  {
    char* lw = at<char>(workspace, L.lists);
    p.ulist = at<int32_t>(lw, L.sl.ulist);
    p.tmask = at<uint4>(lw, L.sl.umask);
    p.ucnt = at<int32_t>(lw, L.sl.ucnt);
    p.usteps = at<int32_t>(lw, L.sl.usteps);
  }
  e = dash::launch_bwd(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "backward");
  return ok();
}

size_t dash_attn_decode_workspace_size(const dash_tensor_t* q, const dash_tensor_t* kcache, int block, int64_t t_cap) {
  if (check_tensor(q, "q") || check_tensor(kcache, "kcache") || (block != 64 && block != 128) ||
      check_group(q->h, kcache->h) || t_cap <= 0)
    return 0;
  return decode_layout(q->b, q->h, kcache->h, q->d, block, t_cap).total;
}

dash_status_t dash_attn_decode_workspace_lists(const dash_tensor_t* q, const dash_tensor_t* kcache, int block,
                                               int64_t t_cap, size_t* idx_offset, size_t* logp_offset,
                                               size_t* cnt_offset) {
  dash_status_t st;
  if ((st = check_tensor(q, "q")) || (st = check_tensor(kcache, "kcache")) || (st = check_group(q->h, kcache->h)))
    return st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (t_cap <= 0) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap must be positive");
  const DecodeLayout L = decode_layout(q->b, q->h, kcache->h, q->d, block, t_cap);
  if (idx_offset) *idx_offset = L.idx;
  if (logp_offset) *logp_offset = L.logp;
  if (cnt_offset) *cnt_offset = L.cnt;
  return ok();
}

dash_status_t dash_attn_decode(const dash_tensor_t* q, const dash_tensor_t* kcache, const dash_tensor_t* vcache,
                               const int32_t* seqlens, const float* summaries, int64_t t_cap, float alpha, int block,
                               dash_tensor_t* out, void* workspace, size_t workspace_bytes, dash_stream_t stream) {
  return dash_attn_decode_ex(q, kcache, vcache, seqlens, summaries, t_cap, alpha, block, out, workspace,
                             workspace_bytes, nullptr, stream);
}

// The decode step once its arguments are checked: dense cache (table null;
// k/v views of [B, Lmax, Hkv, d]) or paged (k/v views of [pages, block, Hkv,
// d], sb = page stride).
static dash_status_t run_decode_step(const dash_tensor_t* q, dash::View kv, dash::View vv, int64_t Hkv, int64_t lmax,
                                     const int32_t* table, int64_t max_blocks, const int32_t* seqlens,
                                     const float* summaries, int64_t t_cap, float alpha, int block, dash_tensor_t* out,
                                     void* workspace, size_t workspace_bytes, float sigma, dash_stream_t stream) {
  const DecodeLayout L = decode_layout(q->b, q->h, Hkv, q->d, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.status), 0, sizeof(dash::DeviceStatus), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(at<char>(workspace, L.n_items), 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  dash::DecodeParams p{};
  p.q = view(q);
  p.k = kv;
  p.v = vv;
  p.block_table = table;
  p.max_blocks = (int)max_blocks;
  p.out = view(out);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.Lmax = (int)lmax;
  p.H = (int)q->h;
  p.Hkv = (int)Hkv;
  p.G = (int)(q->h / Hkv);
  p.D = (int)q->d;
  p.block = block;
  p.alpha = alpha;
  p.seqlens = seqlens;
  p.summaries = summaries;
  p.t_cap = t_cap;
  p.scores = at<float>(workspace, L.scores);
  p.idx = at<int32_t>(workspace, L.idx);
  p.logp = at<float>(workspace, L.logp);
  p.cnt = at<int32_t>(workspace, L.cnt);
  p.items = at<int32_t>(workspace, L.items);
  p.n_items = at<int32_t>(workspace, L.n_items);
  p.pair_base = at<int32_t>(workspace, L.pair_base);
  p.part_o = at<float>(workspace, L.part_o);
  p.part_ml = at<float>(workspace, L.part_ml);
  p.max_items = L.max_items;
  p.chunk_blocks = L.chunk;
  p.sigma = sigma;
  p.c_lo = 0;
  p.c_hi = (int)t_cap;
  p.summ_cap = t_cap;
  p.status = at<dash::DeviceStatus>(workspace, L.status);
  e = dash::launch_decode_route(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode route");
  e = dash::launch_decode_attend(p, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "decode attend");
  return ok();
}

dash_status_t dash_attn_decode_ex(const dash_tensor_t* q, const dash_tensor_t* kcache, const dash_tensor_t* vcache,
                                  const int32_t* seqlens, const float* summaries, int64_t t_cap, float alpha,
                                  int block, dash_tensor_t* out, void* workspace, size_t workspace_bytes,
                                  const dash_options_t* opts, dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if ((st = check_tensor(q, "q")) || (st = check_tensor(kcache, "kcache")) || (st = check_tensor(vcache, "vcache")) ||
      (st = check_tensor(out, "out")) || (st = check_common(alpha, block)) || (st = check_group(q->h, kcache->h)))
    return st;
  if (q->s != 1 || out->s != 1) return fail(DASH_ERR_INVALID_ARGUMENT, "decode takes one query token (s == 1)");
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "decode supports f16 and bf16");
  if (q->dtype != kcache->dtype || q->dtype != vcache->dtype || q->dtype != out->dtype)
    return fail(DASH_ERR_INVALID_ARGUMENT, "q, caches and out must share one dtype");
  if (kcache->b != q->b || vcache->b != q->b || out->b != q->b) return fail(DASH_ERR_INVALID_ARGUMENT, "batch mismatch");
  if (kcache->d != q->d || vcache->d != q->d || out->d != q->d) return fail(DASH_ERR_INVALID_ARGUMENT, "head dim mismatch");
  if (vcache->h != kcache->h || vcache->s != kcache->s) return fail(DASH_ERR_INVALID_ARGUMENT, "kcache and vcache differ");
  if (out->h != q->h) return fail(DASH_ERR_INVALID_ARGUMENT, "out must have q's shape");
  if (!seqlens || !summaries) return fail(DASH_ERR_INVALID_ARGUMENT, "null seqlens or summaries");
  if (reinterpret_cast<uintptr_t>(summaries) % 16) return fail(DASH_ERR_INVALID_ARGUMENT, "summaries not 16-byte aligned");
  const int64_t T = (kcache->s + block - 1) / block;
  if (t_cap < T) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap %lld < ceil(Lmax / block)", (long long)t_cap);
  if (t_cap > 4096) return fail(DASH_ERR_UNSUPPORTED, "t_cap above 4096");
  return run_decode_step(q, view(kcache), view(vcache), kcache->h, kcache->s, nullptr, 0, seqlens, summaries, t_cap,
                         alpha, block, out, workspace, workspace_bytes, sigma, stream);
}

// ------------------------------------------------------------------ paged KV cache

static dash_status_t check_pages(const dash_tensor_t* pages, const char* name, int block, const int32_t* table,
                                 int64_t max_blocks) {
  dash_status_t st;
  if ((st = check_tensor(pages, name))) return st;
  if (pages->s != block) return fail(DASH_ERR_INVALID_ARGUMENT, "%s: page size %lld != block %d", name,
                                     (long long)pages->s, block);
  if (!table || max_blocks < 1) return fail(DASH_ERR_INVALID_ARGUMENT, "null block table or max_blocks < 1");
  return DASH_OK;
}

dash_status_t dash_attn_summarize_paged(const dash_tensor_t* k_pages, const int32_t* block_table, int64_t max_blocks,
                                        int64_t batch, const int32_t* seqlens, const float* w_s, const float* qbar,
                                        int block, float* summaries, int64_t t_cap, int64_t first_block,
                                        dash_stream_t stream) {
  dash_status_t st;
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if ((st = check_pages(k_pages, "k_pages", block, block_table, max_blocks))) return st;
  if (batch < 1 || !seqlens) return fail(DASH_ERR_INVALID_ARGUMENT, "batch < 1 or null seqlens");
  if (!w_s || !summaries) return fail(DASH_ERR_INVALID_ARGUMENT, "null w_s or summaries");
  if (reinterpret_cast<uintptr_t>(summaries) % 16 || reinterpret_cast<uintptr_t>(w_s) % 16 ||
      reinterpret_cast<uintptr_t>(qbar) % 16)
    return fail(DASH_ERR_INVALID_ARGUMENT, "summaries, w_s or qbar not 16-byte aligned");
  if (t_cap < max_blocks) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap < max_blocks");
  if (first_block < 0) return fail(DASH_ERR_INVALID_ARGUMENT, "first_block < 0");
  dash::PoolParams p{};
  p.k = view(k_pages);
  p.dtype = k_pages->dtype;
  p.B = (int)batch;
  p.S = (int)(max_blocks * block);
  p.Hkv = (int)k_pages->h;
  p.D = (int)k_pages->d;
  p.block = block;
  p.seqlens = seqlens;
  p.w_s = w_s;
  p.qbar = qbar;
  p.block_table = block_table;
  p.max_blocks = (int)max_blocks;
  p.summaries = summaries;
  p.t_cap = t_cap;
  p.first_block = first_block;
  cudaError_t e = dash::launch_pool(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "summarize (paged)");
  return ok();
}

dash_status_t dash_attn_decode_paged(const dash_tensor_t* q, const dash_tensor_t* k_pages, const dash_tensor_t* v_pages,
                                     const int32_t* block_table, int64_t max_blocks, const int32_t* seqlens,
                                     const float* summaries, int64_t t_cap, float alpha, int block, dash_tensor_t* out,
                                     void* workspace, size_t workspace_bytes, const dash_options_t* opts,
                                     dash_stream_t stream) {
  dash_status_t st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if ((st = check_tensor(q, "q")) || (st = check_tensor(out, "out")) || (st = check_common(alpha, block))) return st;
  if ((st = check_pages(k_pages, "k_pages", block, block_table, max_blocks)) ||
      (st = check_pages(v_pages, "v_pages", block, block_table, max_blocks)) || (st = check_group(q->h, k_pages->h)))
    return st;
  if (q->s != 1 || out->s != 1) return fail(DASH_ERR_INVALID_ARGUMENT, "decode takes one query token (s == 1)");
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "decode supports f16 and bf16");
  if (q->dtype != k_pages->dtype || q->dtype != v_pages->dtype || q->dtype != out->dtype)
    return fail(DASH_ERR_INVALID_ARGUMENT, "q, pages and out must share one dtype");
  if (k_pages->d != q->d || v_pages->d != q->d || out->d != q->d || v_pages->h != k_pages->h ||
      v_pages->b != k_pages->b)
    return fail(DASH_ERR_INVALID_ARGUMENT, "page shapes do not match q");
  if (out->b != q->b || out->h != q->h) return fail(DASH_ERR_INVALID_ARGUMENT, "out must have q's shape");
  if (!seqlens || !summaries) return fail(DASH_ERR_INVALID_ARGUMENT, "null seqlens or summaries");
  if (reinterpret_cast<uintptr_t>(summaries) % 16) return fail(DASH_ERR_INVALID_ARGUMENT, "summaries not 16-byte aligned");
  if (t_cap < max_blocks) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap < max_blocks");
  if (t_cap > 4096) return fail(DASH_ERR_UNSUPPORTED, "t_cap above 4096");
  return run_decode_step(q, view(k_pages), view(v_pages), k_pages->h, max_blocks * block, block_table, max_blocks,
                         seqlens, summaries, t_cap, alpha, block, out, workspace, workspace_bytes, sigma, stream);
}

// ------------------------------------------------------------------ context-parallel decode

static dash_status_t cp_common(const dash_tensor_t* q, int64_t kv_heads, const int32_t* seqlens, int64_t lmax,
                               int block, int64_t t_cap) {
  dash_status_t st;
  if ((st = check_tensor(q, "q")) || (st = check_group(q->h, kv_heads))) return st;
  if (q->s != 1) return fail(DASH_ERR_INVALID_ARGUMENT, "decode takes one query token (s == 1)");
  if (q->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "context-parallel decode supports f16 and bf16");
  if (block != 64 && block != 128) return fail(DASH_ERR_UNSUPPORTED, "block %d not in {64, 128}", block);
  if (!seqlens || lmax < 1) return fail(DASH_ERR_INVALID_ARGUMENT, "null seqlens or lmax < 1");
  if (t_cap < (lmax + block - 1) / block) return fail(DASH_ERR_INVALID_ARGUMENT, "t_cap < ceil(lmax / block)");
  if (t_cap > 4096) return fail(DASH_ERR_UNSUPPORTED, "t_cap above 4096");
  return DASH_OK;
}

static dash::DecodeParams cp_params(const dash_tensor_t* q, int64_t kv_heads, const int32_t* seqlens, int64_t lmax,
                                    int block, int64_t t_cap) {
  dash::DecodeParams p{};
  p.q = view(q);
  p.dtype = q->dtype;
  p.B = (int)q->b;
  p.Lmax = (int)lmax;
  p.H = (int)q->h;
  p.Hkv = (int)kv_heads;
  p.G = (int)(q->h / kv_heads);
  p.D = (int)q->d;
  p.block = block;
  p.seqlens = seqlens;
  p.t_cap = t_cap;
  p.sigma = 1.0f;
  p.c_lo = 0;
  p.c_hi = (int)t_cap;
  p.summ_cap = t_cap;
  return p;
}

dash_status_t dash_attn_cp_scores(const dash_tensor_t* q, int64_t kv_heads, const float* summaries, int64_t summ_cap,
                                  int64_t block_lo, int64_t block_hi, const int32_t* seqlens, int64_t lmax, float alpha,
                                  int block, float* scores, int64_t t_cap, dash_stream_t stream) {
  dash_status_t st;
  if ((st = cp_common(q, kv_heads, seqlens, lmax, block, t_cap)) || (st = check_common(alpha, block))) return st;
  if (!summaries || !scores) return fail(DASH_ERR_INVALID_ARGUMENT, "null summaries or scores");
  if (reinterpret_cast<uintptr_t>(summaries) % 16) return fail(DASH_ERR_INVALID_ARGUMENT, "summaries not 16-byte aligned");
  if (block_lo < 0 || block_hi < block_lo || block_hi - block_lo > summ_cap || block_hi > t_cap)
    return fail(DASH_ERR_INVALID_ARGUMENT, "bad block range [%lld, %lld) for summ_cap %lld",
                (long long)block_lo, (long long)block_hi, (long long)summ_cap);
  dash::DecodeParams p = cp_params(q, kv_heads, seqlens, lmax, block, t_cap);
  p.alpha = alpha;
  p.summaries = summaries;
  p.summ_cap = summ_cap;
  p.c_lo = (int)block_lo;
  p.c_hi = (int)block_hi;
  p.scores = scores;
  cudaError_t e = dash::launch_cp_scores(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "context-parallel scores");
  return ok();
}

dash_status_t dash_attn_cp_lists(const dash_tensor_t* q, int64_t kv_heads, const float* scores, const int32_t* seqlens,
                                 int64_t lmax, float alpha, int block, int32_t* idx, float* logp, int32_t* cnt,
                                 int64_t t_cap, dash_stream_t stream) {
  dash_status_t st;
  if ((st = cp_common(q, kv_heads, seqlens, lmax, block, t_cap)) || (st = check_common(alpha, block))) return st;
  if (!scores || !idx || !logp || !cnt) return fail(DASH_ERR_INVALID_ARGUMENT, "null scores or lists");
  dash::DecodeParams p = cp_params(q, kv_heads, seqlens, lmax, block, t_cap);
  p.alpha = alpha;
  p.scores = const_cast<float*>(scores);
  p.idx = idx;
  p.logp = logp;
  p.cnt = cnt;
  cudaError_t e = dash::launch_cp_lists(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "context-parallel lists");
  return ok();
}

dash_status_t dash_attn_cp_attend(const dash_tensor_t* q, const dash_tensor_t* kshard, const dash_tensor_t* vshard,
                                  int64_t tok_lo, const int32_t* seqlens, int64_t lmax, const int32_t* idx,
                                  const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                  const dash_options_t* opts, float* part, dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_tensor(kshard, "kshard")) || (st = check_tensor(vshard, "vshard"))) return st;
  if ((st = cp_common(q, kshard->h, seqlens, lmax, block, t_cap))) return st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if (q->dtype != kshard->dtype || q->dtype != vshard->dtype) return fail(DASH_ERR_INVALID_ARGUMENT, "dtype mismatch");
  if (kshard->b != q->b || vshard->b != q->b || kshard->d != q->d || vshard->d != q->d || vshard->h != kshard->h ||
      vshard->s != kshard->s)
    return fail(DASH_ERR_INVALID_ARGUMENT, "shard shapes do not match q");
  if (tok_lo < 0 || tok_lo % block || kshard->s % block)
    return fail(DASH_ERR_INVALID_ARGUMENT, "shard start and length must be multiples of the block");
  if (!idx || !logp || !cnt || !part) return fail(DASH_ERR_INVALID_ARGUMENT, "null lists or partials");
  dash::DecodeParams p = cp_params(q, kshard->h, seqlens, lmax, block, t_cap);
  p.k = view(kshard);
  p.v = view(vshard);
  p.sigma = sigma;
  p.idx = const_cast<int32_t*>(idx);
  p.logp = const_cast<float*>(logp);
  p.cnt = const_cast<int32_t*>(cnt);
  p.tok_lo = (int)tok_lo;
  p.tok_n = (int)kshard->s;
  p.part = part;
  cudaError_t e = dash::launch_cp_attend(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "context-parallel attention");
  return ok();
}

// Workspace of the split-KV shard attention: per (b, g) the shard's entry
// range, the work items and their per-item partials.
struct CpAttendLayout {
  size_t shard, items, n_items, pair_base, part_o, part_ml, total;
  int64_t max_items;
  int chunk;
};

static CpAttendLayout cp_attend_layout(int64_t B, int64_t H, int64_t Hkv, int64_t D, int block, int64_t t_cap) {
  CpAttendLayout L{};
  const int64_t G = H / Hkv;
  L.chunk = block == 64 ? 16 : 8;
  L.max_items = dash::decode_max_items(B, Hkv, t_cap, L.chunk);
  size_t off = 0;
  L.shard = off;
  off = align256(off + (size_t)B * Hkv * 4 * 4);
  L.items = off;
  off = align256(off + (size_t)L.max_items * 2 * 4);
  L.n_items = off;
  off = align256(off + 4);
  L.pair_base = off;
  off = align256(off + (size_t)B * Hkv * 4);
  L.part_o = off;
  off = align256(off + (size_t)L.max_items * G * D * 4);
  L.part_ml = off;
  off = align256(off + (size_t)L.max_items * G * 2 * 4);
  L.total = off;
  return L;
}

size_t dash_attn_cp_attend_workspace_size(int64_t batch, int64_t heads, int64_t kv_heads, int64_t head_dim, int block,
                                          int64_t t_cap) {
  if (batch < 1 || kv_heads < 1 || heads < kv_heads || heads % kv_heads || head_dim < 1 || block < 1 || t_cap < 1)
    return 0;
  return cp_attend_layout(batch, heads, kv_heads, head_dim, block, t_cap).total;
}

dash_status_t dash_attn_cp_attend_ex(const dash_tensor_t* q, const dash_tensor_t* kshard, const dash_tensor_t* vshard,
                                     int64_t tok_lo, const int32_t* seqlens, int64_t lmax, const int32_t* idx,
                                     const float* logp, const int32_t* cnt, int64_t t_cap, int block,
                                     const dash_options_t* opts, float* part, void* workspace, size_t workspace_bytes,
                                     dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_tensor(kshard, "kshard")) || (st = check_tensor(vshard, "vshard"))) return st;
  if ((st = cp_common(q, kshard->h, seqlens, lmax, block, t_cap))) return st;
  float sigma;
  const float* qbar;
  if ((st = read_options(opts, false, &sigma, &qbar))) return st;
  if (q->dtype != kshard->dtype || q->dtype != vshard->dtype) return fail(DASH_ERR_INVALID_ARGUMENT, "dtype mismatch");
  if (kshard->b != q->b || vshard->b != q->b || kshard->d != q->d || vshard->d != q->d || vshard->h != kshard->h ||
      vshard->s != kshard->s)
    return fail(DASH_ERR_INVALID_ARGUMENT, "shard shapes do not match q");
  if (tok_lo < 0 || tok_lo % block || kshard->s % block)
    return fail(DASH_ERR_INVALID_ARGUMENT, "shard start and length must be multiples of the block");
  if (!idx || !logp || !cnt || !part) return fail(DASH_ERR_INVALID_ARGUMENT, "null lists or partials");
  const CpAttendLayout L = cp_attend_layout(q->b, q->h, kshard->h, q->d, block, t_cap);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(DASH_ERR_INVALID_ARGUMENT, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < L.total)
    return fail(DASH_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(at<char>(workspace, L.n_items), 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  dash::DecodeParams p = cp_params(q, kshard->h, seqlens, lmax, block, t_cap);
  p.k = view(kshard);
  p.v = view(vshard);
  p.sigma = sigma;
  p.idx = const_cast<int32_t*>(idx);
  p.logp = const_cast<float*>(logp);
  p.cnt = const_cast<int32_t*>(cnt);
  p.tok_lo = (int)tok_lo;
  p.tok_n = (int)kshard->s;
  p.part = part;
  p.shard = at<int32_t>(workspace, L.shard);
  p.items = at<int32_t>(workspace, L.items);
  p.n_items = at<int32_t>(workspace, L.n_items);
  p.pair_base = at<int32_t>(workspace, L.pair_base);
  p.part_o = at<float>(workspace, L.part_o);
  p.part_ml = at<float>(workspace, L.part_ml);
  p.max_items = L.max_items;
  p.chunk_blocks = L.chunk;
  e = dash::launch_cp_attend_mma(p, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "context-parallel attention (split-KV)");
  return ok();
}

dash_status_t dash_attn_cp_merge(const float* parts, int64_t n_parts, dash_tensor_t* out, dash_stream_t stream) {
  dash_status_t st;
  if ((st = check_tensor(out, "out"))) return st;
  if (out->s != 1) return fail(DASH_ERR_INVALID_ARGUMENT, "out must be [B, 1, H, d]");
  if (out->dtype == DASH_F32) return fail(DASH_ERR_UNSUPPORTED, "context-parallel decode supports f16 and bf16");
  if (!parts || n_parts < 1) return fail(DASH_ERR_INVALID_ARGUMENT, "null parts or n_parts < 1");
  cudaError_t e = dash::launch_cp_merge(parts, (int)n_parts, (int)out->b, (int)out->h, (int)out->d, view(out),
                                        out->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "context-parallel merge");
  return ok();
}

dash_status_t dash_attn_lists_to_mask(const int32_t* idx, const int32_t* cnt, int64_t rows, int64_t t_cap,
                                      uint32_t* mask, int64_t n_words, dash_stream_t stream) {
  if (rows < 0 || t_cap <= 0) return fail(DASH_ERR_INVALID_ARGUMENT, "rows < 0 or t_cap <= 0");
  if (rows > 0 && (!idx || !cnt || !mask)) return fail(DASH_ERR_INVALID_ARGUMENT, "null idx, cnt or mask");
  if (n_words * 32 < t_cap) return fail(DASH_ERR_INVALID_ARGUMENT, "n_words * 32 < t_cap");
  if (n_words > 128) return fail(DASH_ERR_UNSUPPORTED, "more than 4096 blocks per row");
  cudaError_t e = dash::launch_lists_to_mask(idx, cnt, rows, t_cap, mask, (int)n_words, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "lists to mask");
  return ok();
}

dash_status_t dash_attn_get_device_status(void* workspace, dash_stream_t stream) {
  if (!workspace) return fail(DASH_ERR_INVALID_ARGUMENT, "null workspace");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  dash::DeviceStatus st{};
  e = cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (st.code == 0) return ok();
  return fail((dash_status_t)st.code, "device reported status %d (detail %d)", st.code, st.detail);
}

}  // extern "C"
