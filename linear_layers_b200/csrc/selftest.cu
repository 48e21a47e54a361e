// selftest.cu — a device-side check of the bounded mbarrier wait.
//
// One CTA initialises an mbarrier that expects one arrival, never arrives,
// and waits on it with mbar_wait_bounded.  The wait must give up after the
// limit and the kernel must record TP_DEVERR_TIMEOUT and return: this is
// the path every pipeline wait in the library takes when its partner never
// signals.
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpl {
namespace {

__global__ void wait_timeout_kernel(int32_t* dev_status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int no_abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    no_abort = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(&bar, 0, limit_ns, &no_abort)) atomicOr(dev_status, TP_DEVERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace tpl

extern "C" tp_status tp_selftest_wait_timeout(int32_t* dev_status, uint32_t limit_us,
                                              void* stream) {
  using namespace tpl;
  if (!dev_status) return TP_ERR_NULL;
  if (limit_us == 0 || limit_us > 10000000u) return TP_ERR_SHAPE;
  if (tp_status s = require_sm100()) return s;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_status, static_cast<uint64_t>(limit_us) * 1000ull);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

extern "C" tp_status tp_debug_stall_next_gemm(int32_t unit, int32_t kblock, uint32_t wait_limit_us) {
  using namespace tpl;
  if (unit < 0 || kblock < 0) return TP_ERR_SHAPE;
  if (wait_limit_us == 0 || wait_limit_us > 10000000u) return TP_ERR_SHAPE;
  arm_gemm_injection(unit, kblock, static_cast<uint64_t>(wait_limit_us) * 1000ull);
  return TP_OK;
}
