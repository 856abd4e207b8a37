// Self-test of the failure-detection path: a one-CTA kernel waits on an
// mbarrier that nothing will ever arrive at.  The wait is the same bounded
// wait every tensor-core kernel uses; it gives up after `limit` cycles, and
// the kernel records SSA_ERR_TIMEOUT in the device status word and returns,
// exactly as a stuck kernel of this library would.  Nothing faults or hangs.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

__global__ void selftest_timeout_kernel(int32_t* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);  // expects one arrival; none will come
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = sm100::mbar_wait(&bar, 0, &abort_flag, limit);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicCAS(status, 0, (int)SSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_timeout(int32_t* status, long long limit_cycles, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(status, limit_cycles);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ssa
