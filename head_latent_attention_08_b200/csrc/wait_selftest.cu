// wait_selftest.cu -- a diagnostic kernel for the bounded device waits of the tensor-core kernels.
//
// One CTA allocates tensor memory, waits on an mbarrier that nothing ever completes through the
// same bounded wait the decode and GEMM kernels use, and, once the wait limit has run out, releases
// its tensor memory and returns. The status word then holds MLA_ERR_TIMEOUT. This gives a test a wait
// that certainly runs out, without a fault, a trap or an endless loop.
#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

__global__ void __launch_bounds__(128) wait_selftest_kernel(int* status, uint64_t wait_ns) {
  __shared__ __align__(8) uint64_t never;      // expects one arrival that no thread makes
  __shared__ uint32_t tmem_slot;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(&tmem_slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) (void)mbar_wait(&never, 0, wait_ns, status);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, 32);
  }
}

int wait_selftest_launch(cudaStream_t s) {
  wait_selftest_kernel<<<1, 128, 0, s>>>(device_status_ptr(), (uint64_t)wait_limit());
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

}  // namespace mla
