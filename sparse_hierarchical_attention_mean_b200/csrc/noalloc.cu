// dash_attn_decode_noalloc: the decode step with its scratch memory in a
// fixed, library-owned device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: code that runs inside
// another engine's execution hook (an inference-server or graph-runtime
// plugin) where allocating device memory is not allowed or would stall the
// device, and programs that fix their whole device-memory budget at start-up
// and may not call cudaMalloc afterwards.  This entry point needs only the
// inputs and outputs.  Its scratch is one file-scope __device__ array of
// kScratchBytes bytes that every GPU which loads this library holds until
// the process exits.  Problems whose decode workspace would exceed it are
// rejected before anything is launched.
//
// The array is shared by every call on a device and keeps the last call's
// contents.  The decode path clears what must start at zero (its status
// word and work-item counter) at the start of every call and writes every
// other scratch entry before reading it.  Two calls whose GPU work overlaps
// (on different streams, or from different host threads without ordering)
// race on the array and give wrong results.
//
// Set-up: the first call on each device looks up the array's device address
// with cudaGetSymbolAddress (with that device current); that first call
// should therefore come before any stream capture.  The address stays valid
// for the life of the device's context: after cudaDeviceReset (or anything
// else that destroys the primary context) the module is loaded again at
// another address, so a process that resets a device must not call this
// entry point (or dash_attn_decode_noalloc_status) on it again.
//
// The status word of a call (a seqlens entry out of range, a bounded device
// wait that gave up) sits at the start of the array;
// dash_attn_decode_noalloc_status reads it without allocating.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dashattn.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" dash_status_t dash_attn_decode_noalloc(const dash_tensor_t* q, const dash_tensor_t* kcache,
                                                  const dash_tensor_t* vcache, const int32_t* seqlens,
                                                  const float* summaries, int64_t t_cap, float alpha, int block,
                                                  dash_tensor_t* out, dash_stream_t stream) {
  const size_t need = dash_attn_decode_workspace_size(q, kcache, block, t_cap);
  if (need == 0) {
    // rejected arguments: the regular entry point reports the precise error
    // from its host-side checks and launches nothing
    return dash_attn_decode(q, kcache, vcache, seqlens, summaries, t_cap, alpha, block, out, nullptr, 0, stream);
  }
  if (need > kScratchBytes) {
    return dash::set_last_error(DASH_ERR_UNSUPPORTED,
                                "dash_attn_decode_noalloc: this problem needs %zu bytes of scratch, the fixed "
                                "scratch array holds %zu; use dash_attn_decode with a workspace",
                                need, kScratchBytes);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return dash::set_last_error(DASH_ERR_CUDA, "dash_attn_decode_noalloc: no usable current device");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess || !p)
        return dash::set_last_error(DASH_ERR_CUDA, "dash_attn_decode_noalloc: scratch address lookup failed: %s",
                                    cudaGetErrorString(e));
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return dash_attn_decode(q, kcache, vcache, seqlens, summaries, t_cap, alpha, block, out, scratch,
                          kScratchBytes, stream);
}

extern "C" dash_status_t dash_attn_decode_noalloc_status(dash_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return dash::set_last_error(DASH_ERR_CUDA, "dash_attn_decode_noalloc_status: no usable current device");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    scratch = g_scratch_addr[dev];
  }
  if (!scratch)
    return dash::set_last_error(DASH_ERR_INVALID_ARGUMENT,
                                "dash_attn_decode_noalloc_status: no dash_attn_decode_noalloc call on this device yet");
  return dash_attn_get_device_status(scratch, stream);
}
