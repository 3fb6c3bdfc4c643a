// Self-test of the bounded-wait path (no counterpart on the pages; it serves
// failure detection without a GPU fault).  One thread waits on an mbarrier
// that nothing arrives at, with the library's own bounded wait; when the
// limit runs out it raises QLORA_ERR_TIMEOUT in the caller's status word and
// the kernel returns, so the context stays usable and the host learns of the
// failure from the status word, exactly as a production kernel's timeout.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

__global__ void bounded_wait_selftest_kernel(int32_t* d_status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival would complete phase 0; none comes
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_for(&bar, 0, limit_ns)) raise_status(d_status, QLORA_ERR_TIMEOUT);
}

cudaError_t launch_bounded_wait_selftest(int32_t* d_status, uint64_t limit_ns, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(d_status, limit_ns);
  return cudaGetLastError();
}

}  // namespace qnf4
