// Self-test of the bounded device waits every kernel of this library uses:
// a producer warp that issues nothing, a consumer warp waiting on the stage
// barrier it would have completed.  The consumer's wait runs out after the
// given limit, the CTA records MOE_Q4_ETIMEOUT in the status word through the
// same teardown as the layer's kernels, and the kernel returns: no trap, no
// hang, the context stays usable.  Test support, not part of the layer.
#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "sm100.cuh"

namespace q4 {

using namespace sm100;

__global__ void __launch_bounds__(64) selftest_wait_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t full;
  __shared__ int abort_flag;
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&full, 1);
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 1) {
    // consumer: waits for a stage nobody produces
    if (!mbar_wait_warp(&full, 0, abort, limit_ns) && threadIdx.x == 32) {
      // (the vote already set the abort flag)
    }
  }
  // producer (warp 0): issues nothing
  __syncthreads();
  if (threadIdx.x == 0 && *abort) record_error(status, MOE_Q4_ETIMEOUT);
}

}  // namespace q4

using namespace q4;

extern "C" int moe_q4_selftest_wait(int32_t* status, unsigned limit_us, void* stream) {
  if (!status || limit_us == 0 || limit_us > 2000000u) return MOE_Q4_EINVAL;
  selftest_wait_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(status, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
