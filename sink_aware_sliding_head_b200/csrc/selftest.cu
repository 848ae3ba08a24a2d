// selftest.cu - device check of failure detection without a GPU fault.
//
// Every pipelined kernel waits on mbarriers through mbar_wait, which gives up
// after a limit of SM clock cycles, records a timeout bit in the status word
// and lets the kernel unwind and exit. This kernel runs that same wait on a
// barrier whose phase completes only when asked to: with nothing arriving the
// wait must run out and report; with the arrival made first it must pass.
#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(long long limit, int arrive_first,
                                                           int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (arrive_first && threadIdx.x == 0) mbar_arrive(smem_u32(&bar));
  __syncthreads();
  const WaitCtx w{abort_flag, status, kStatusTimeoutSelftest};
  const bool done = mbar_wait_warp(smem_u32(&bar), 0, w, limit);
  if (threadIdx.x == 0) status[1] = done ? 1 : 0;
}

}  // namespace

cudaError_t launch_wait_selftest(long long limit, int arrive_first, int* status,
                                 cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(limit, arrive_first, status);
  return cudaGetLastError();
}

}  // namespace flint
