// wkv4_bwd_noalloc.cu -- wkv4_backward_noalloc: the RWKV-4 backward for callers
// that cannot hand the library a workspace.
//
// wkv4_backward needs a device workspace (per-lane gw/gu partial sums, and the
// state checkpoints when the caller has none). Some callers cannot allocate
// device memory per call: code reached through a plain C interface that only
// receives the tensors it must read and write (no allocator behind it), and
// latency-critical loops that must not call cudaMalloc/cudaFree (they are slow
// and can synchronise the device) or that run under a fixed memory budget.
// This entry point runs the same kernels with the workspace placed in a
// file-scope device array instead.
//
// The array is kNoallocScratchBytes (4 MiB) and lives on every GPU that loads
// the library until the process exits. The call uses the array of the current
// device (which must own the tensors and the stream); its device address is
// looked up once per device, with that device current, on the first call made
// on it (so make that first call before any stream capture). Every call shares
// the array: calls whose kernels overlap on the GPU (several streams, or
// several host threads) race on it and must be serialised by the caller.
// Nothing in it has to start at zero: each call's kernels write every scratch
// element before reading it (the backward writes its partial sums even after a
// copy wait that gave up, as zeros; such a call's results are undefined and
// the device error word says so).
#include <cuda_runtime.h>

#include <mutex>

#include "wkv.h"
#include "wkv_internal.h"

#define WKV_EXPORT extern "C" __attribute__((visibility("default")))

namespace wkv {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

wkv_status noalloc_fail(wkv_status s, const char* why) {
  set_last_error(why);
  return s;
}

// Device address of g_noalloc_scratch on the current device. The host-side
// name of the array is only a stand-in, never a device address.
wkv_status scratch_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(WKV_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
      return noalloc_fail(WKV_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch) failed");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return WKV_OK;
}

}  // namespace
}  // namespace wkv

using namespace wkv;

WKV_EXPORT wkv_status wkv4_backward_noalloc(int64_t B, int64_t T, int64_t C, int dtype, const float* w,
                                            const float* u, const void* k, const void* v, const void* gy,
                                            const float* ckpt, void* gk, void* gv, float* gw, float* gu,
                                            void* stream) {
  const size_t need = wkv4_backward_workspace_bytes(B, T, C, ckpt != nullptr);
  if (need > kNoallocScratchBytes)
    return noalloc_fail(WKV_ERR_UNSUPPORTED,
                        "wkv4_backward_noalloc: wkv4_backward_workspace_bytes() of the problem exceeds the 4 MiB "
                        "static array; pass ckpt or use wkv4_backward");
  void* scratch = nullptr;
  if (B > 0 && T > 0 && C > 0) {
    if (wkv_status s = scratch_ptr(&scratch)) return s;
  }
  // The workspace entry point does every argument check and launch; it only
  // receives the static array as its workspace.
  return wkv4_backward(B, T, C, dtype, w, u, k, v, gy, ckpt, gk, gv, gw, gu, scratch, kNoallocScratchBytes,
                       stream);
}
