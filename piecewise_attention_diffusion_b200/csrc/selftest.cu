// bsa_selftest_wait_timeout: the failure path shared by the library's kernels, run
// without a fault. Every wait in the kernels is sm100::mbar_wait, bounded by
// %globaltimer: when it runs out it raises the CTA's abort flag, the kernel leaves its
// loops, and BSA_ERR_TIMEOUT is written to the status word. Here one thread waits on an
// mbarrier that nothing ever arrives on, so the wait must run out after timeout_ns.
#include "../../include/bsattn.h"
#include "common.cuh"
#include "sm100.cuh"

namespace bsa {
namespace {

__global__ void k_wait_selftest(int32_t* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // no thread or copy ever arrives on `bar`, so phase 0 never completes
    const bool ok = sm100::mbar_wait(&bar, 0, &abort_sh, timeout_ns);
    if (!ok && abort_sh) report(status, BSA_ERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace bsa

extern "C" BSA_API bsa_status bsa_selftest_wait_timeout(int64_t timeout_ns, int32_t* status,
                                                        void* stream) {
  if (status == nullptr || timeout_ns < 1 || timeout_ns > 10000000000ll)
    return BSA_ERR_INVALID_ARG;
  bsa::k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      status, static_cast<uint64_t>(timeout_ns));
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}
