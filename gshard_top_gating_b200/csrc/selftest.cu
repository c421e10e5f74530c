// selftest.cu -- a kernel whose bounded mbarrier wait is made to run out.
//
// It initialises an mbarrier that nothing will ever arrive on and waits for it
// with the same bounded-wait helper the tensor-core kernels use.  The wait gives
// up after limit_ns, sets DEVERR_TIMEOUT in the error word and returns, so the
// host sees a timeout status and the context stays usable.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

__global__ void wait_selftest_kernel(unsigned* flag, unsigned* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(b, 0, err, limit_ns);
    flag[0] = ok ? 1u : 2u;
  }
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned* flag, unsigned* err, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(flag, err, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
