// selfcheck.cu -- the failure path of the bounded waits, on demand.
//
// Every wait of the kernels on a TMA copy (an mbarrier phase) is bounded: if
// the phase never completes, the wait gives up after its limit, records
// WKV_DEVERR_WAIT_TIMEOUT in the device error word and the kernel returns,
// so the context stays usable and the host learns of it through
// wkv_device_error(). This kernel takes that path deliberately: one warp
// waits on a barrier that nothing will complete, with a short limit.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

__global__ void __launch_bounds__(32) wkv_wait_selfcheck_kernel(uint64_t limit_ns, unsigned* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  const uint64_t t0 = globaltimer_ns();
  bool done = mbar_try_wait(&bar, 0);  // phase 0 never completes: no thread arrives
  while (!done) {
    done = mbar_try_wait_sleep(&bar, 0, 1000u);
    if (!done && globaltimer_ns() - t0 > limit_ns) {
      if (threadIdx.x == 0) record_error(err, WKV_DEVERR_WAIT_TIMEOUT);
      break;
    }
  }
}

wkv_status launch_wait_selfcheck(int64_t limit_ns, cudaStream_t stream, unsigned* err, const char** why) {
  wkv_wait_selfcheck_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ns, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv_wait_selfcheck kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
