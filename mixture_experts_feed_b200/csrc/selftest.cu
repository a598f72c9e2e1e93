// Self-test of the stall detection every pipeline wait relies on.
//
// One block waits, through the same bounded mbarrier wait the grouped GEMM
// uses (sm100_ptx.cuh), on a barrier nothing ever arrives on.  After the
// given limit the wait gives up, records DEV_WAIT_TIMEOUT in the workspace
// status word and the kernel returns: the GPU is never hung and the CUDA
// context stays usable, which the caller can then check.
#include <cuda_runtime.h>

#include "common.cuh"
#include "inkling_moe.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);   // expects one arrival that never comes
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = sm100::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    if (ok) record_status(status, DEV_BAD_ROW);   // impossible: flag the test as broken
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                  uint32_t limit_ms, void* stream) {
  if (workspace == nullptr || workspace_bytes < 256 || limit_ms == 0 || limit_ms > 10000)
    return MOE_ERR_INVALID_ARG;
  moe::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<int32_t*>(workspace), static_cast<uint64_t>(limit_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
