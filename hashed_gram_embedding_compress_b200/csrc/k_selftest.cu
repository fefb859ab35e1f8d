// Self-test of the bounded-wait path shared by the tensor-core kernels: a
// one-CTA kernel waits on an mbarrier that nothing ever arrives at.  The wait
// gives up after kWaitLimitNs, records kDevErrTimeout in the error word and
// the kernel returns normally; the context stays usable.
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

__global__ void wait_timeout_kernel(unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: no thread arrives
    wait_ready(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), err);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* err, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace engram
