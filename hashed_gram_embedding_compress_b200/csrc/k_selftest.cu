// Self-test of the bounded waits shared by the tensor-core kernels: a
// one-CTA kernel waits on an mbarrier that nothing ever arrives at (which = 0),
// or on a count in global memory that never reaches its target (which = 1,
// the wait of the one-launch short-call kernel).  The wait gives up after
// kWaitLimitNs, records kDevErrTimeout in the error word and the kernel
// returns normally; the context stays usable.
#include "sm100_ptx.cuh"
#include "sm100_wait.cuh"

namespace engram {

namespace {

using namespace sm100;

__device__ unsigned g_never_counted = 0;  // no thread ever adds to it

__global__ void wait_timeout_kernel(unsigned* err, int which) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* abort = reinterpret_cast<volatile int*>(&abort_flag);
    if (which == 0)
      wait_ready(smem_u32(&bar), 0, abort, err);  // phase 0 never completes
    else
      wait_count(&g_never_counted, 1u, abort, err);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* err, int which, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err, which);
  return cudaGetLastError();
}

}  // namespace engram
