// Self-test of the bounded device waits that every kernel of the library uses.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits for it through
// the same Waiter as the kernels (a bounded number of try_wait rounds). The wait gives
// up, sets its bit in the caller's error word and the kernel returns: the path a kernel
// takes when a TMA load or a tensor-core commit never completes, exercised without
// breaking any real producer. Nothing faults, traps or spins without bound.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace sa {

__global__ void wait_selftest_kernel(int32_t* err_flag, uint32_t rounds, int32_t* waited) {
  __shared__ __align__(8) uint64_t never;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    tc::mbar_init(smem_u32(&never), 1);
    abort_word = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tc::Waiter wt{&abort_word, err_flag, rounds};
    const bool ok = wt.wait(smem_u32(&never), 0, 0);
    *waited = ok ? 1 : 0;  // 0: the wait gave up, as it must
  }
}

cudaError_t launch_wait_selftest(int32_t* err_flag, uint32_t rounds, int32_t* waited,
                                 cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err_flag, rounds, waited);
  return cudaGetLastError();
}

}  // namespace sa
