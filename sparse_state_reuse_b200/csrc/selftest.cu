// Failure-detection self-test: one thread waits, with a time limit, on a
// barrier that nothing will ever complete.  The bounded wait gives up,
// records DITANGO_ERR_TIMEOUT in the caller's status word and the kernel
// returns normally -- the same path a stalled pipeline stage takes in the
// attention kernel.  Nothing faults, traps or hangs.
#include "common.cuh"

namespace ditango {

__global__ void bounded_wait_selftest_kernel(long long limit_ns, int *dev_status) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl ctl{&abort_flag, dev_status, limit_ns};
    if (wait_bounded(smem_u32(&bar), 0, ctl)) atomicExch(dev_status, (int)DITANGO_OK);
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(smem_u32(&bar));  // leave the barrier completed
}

cudaError_t launch_bounded_wait_selftest(long long limit_ns, int *dev_status, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, dev_status);
  return cudaGetLastError();
}

}  // namespace ditango
