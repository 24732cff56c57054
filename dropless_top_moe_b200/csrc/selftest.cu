// Diagnostics: the bounded pipeline wait on a barrier that never completes.
//
// Every mbarrier wait of the tcgen05 GEMM pipelines is bounded: after a time
// limit the waiting thread raises the kernel's abort flag, sets
// MOE_DEVERR_TIMEOUT in the caller's status word and returns, so a stalled
// pipeline ends the kernel with an error the host can read instead of hanging
// the GPU.  moe_selftest_wait_timeout runs that same wait (mbar_wait_bounded)
// in one block on a barrier nothing ever arrives at, with a caller-chosen
// limit, so the failure path can be exercised without a fault.
#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace {

using namespace moe::umma;

__global__ void wait_timeout_kernel(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    abort_flag = 0;
  }
  __syncthreads();
  // one arrival expected, none made: only the time limit ends this wait
  if (threadIdx.x == 0) (void)mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, status, timeout_ns);
}

}  // namespace

extern "C" moe_status moe_selftest_wait_timeout(int32_t* status, int64_t timeout_ns, moe_stream_t stream) {
  if (!status || timeout_ns < 1000 || timeout_ns > 1000000000) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRACED("selftest_wait_timeout", s, (wait_timeout_kernel<<<1, 32, 0, s>>>((int*)status, (uint64_t)timeout_ns)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}
