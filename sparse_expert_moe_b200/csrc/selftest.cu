// selftest.cu -- exercises the bounded-wait path every tcgen05 kernel relies on to
// return instead of hanging: one warp waits on an mbarrier that nothing arrives on,
// gives up after its clock budget, records MOE_ERR_TIMEOUT in the status word and
// raises the CTA abort flag; a second warp, waiting on another barrier that nothing
// completes, leaves through that flag.  No trap, no fault: the context stays usable.
#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void bounded_wait_kernel(int* status, long long budget_cycles) {
  __shared__ uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    // phase 0 of bars[0] never completes: the budget runs out
    mbar_wait_budget(&bars[0], 0, ab, status, budget_cycles);
  } else {
    // an effectively unbounded budget: only the abort flag ends this wait
    mbar_wait_budget(&bars[1], 0, ab, status, budget_cycles * 1000);
  }
  __syncthreads();
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_bounded_wait(void* ws, long long budget_cycles,
                                                cudaStream_t stream) {
  if (!ws || budget_cycles <= 0 || budget_cycles > (1LL << 33)) return MOE_ERR_INVALID_ARG;
  moe::bounded_wait_kernel<<<1, 64, 0, stream>>>(static_cast<int*>(ws), budget_cycles);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
