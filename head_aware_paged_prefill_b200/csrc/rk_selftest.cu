// Diagnostic: one CTA whose thread waits on a shared-memory mbarrier that
// nothing ever completes, through the same bounded wait the attention kernel
// uses.  When the limit runs out the wait raises RK_DEV_TIMEOUT in the given
// word and the kernel returns normally: the timeout path is exercised on the
// device without a fault, a trap or a hang.
#include <cuda_runtime.h>

#include "rk_internal.h"
#include "sm100.cuh"

namespace rk {

__global__ void selftest_wait_kernel(int* word, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ int site;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    site = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{&abort_flag, word, &site};
    mbar_wait(&bar, 0, wc, 99, limit_ns);  // nothing arrives: gives up after limit_ns
  }
}

cudaError_t launch_selftest_wait(int* word, int wait_ms, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(word, static_cast<uint64_t>(wait_ms) * 1000000ull);
  return cudaGetLastError();
}

}  // namespace rk
