// Self-test of the bounded-wait path shared by the pipelined kernels.
#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

// One warp waits on an mbarrier that nothing ever arrives on.  The wait can
// only run out; the kernel then records NABLA_ERR_TIMEOUT in the status word
// exactly as the attention kernels do when one of their waits runs out.
__global__ void wait_selftest_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = sm100::mbar_wait(&bar, 0, (volatile int*)&abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace nabla
