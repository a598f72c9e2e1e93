// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory.  Some callers do not own the device allocator: a plugin inside an
// inference engine whose enqueue step must not allocate because the engine
// plans every byte of device memory ahead of time, or a process running
// under a fixed device-memory budget where a cudaMalloc may fail or stall.
// Such a caller cannot hand moe_permute a workspace, so this entry point
// keeps the one scratch buffer the permutation needs (its per-expert row
// counters) in a file-scope __device__ array instead.  The caller still
// passes every input and output buffer.
//
// Properties of the static scratch:
//   - it holds kNoAllocMaxExperts int32 counters (4 KiB); every GPU that loads
//     this library keeps it resident until the process exits;
//   - every call shares it and it keeps the last call's contents, so each
//     call clears the counters on its stream before counting;
//   - two calls whose kernels overlap on the GPU (different streams, or
//     different host threads) race on it and produce garbage: order them.
// No cudaMalloc, cudaFree or allocating library routine is called here.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "inkling_moe.h"
#include "internal.h"

namespace moe {
namespace {

constexpr int kNoAllocMaxExperts = 1024;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocMaxExperts];

// Device address of g_permute_scratch, looked up once per device and kept
// for the life of the process (so no cudaDeviceReset between calls).  In
// host code the name g_permute_scratch is a host-side stand-in, not a device
// address, so it must never be passed to a kernel.
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

moe_status_t scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const moe_layer_desc_t* desc, const int32_t* topk_idx,
                                            const uint8_t* padding_mask, const void* x,
                                            int32_t* expert_offsets, int32_t* perm_slot,
                                            int32_t* inv_perm, void* x_perm, void* stream) {
  using namespace moe;
  Layer L;
  const moe_status_t st = validate_desc(desc, &L);
  if (st != MOE_OK) return st;
  if (L.E > kNoAllocMaxExperts) return MOE_ERR_UNSUPPORTED;
  // as moe_permute: x_perm null means no row copy (x is then not read)
  if (topk_idx == nullptr || expert_offsets == nullptr || perm_slot == nullptr ||
      inv_perm == nullptr ||
      (x_perm != nullptr && (x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15) != 0 ||
                             (reinterpret_cast<uintptr_t>(x_perm) & 15) != 0)))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L.T == 0)
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (L.E + 1), s) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  int32_t* counts = nullptr;
  const moe_status_t sc = scratch_for_current_device(&counts);
  if (sc != MOE_OK) return sc;
  // launch_permute clears the counters on `s` before counting.  With no
  // workspace there is no status word: an out-of-range expert id is skipped
  // (its slot gets inv_perm = -1) without being reported.
  const cudaError_t e = launch_permute(L, topk_idx, padding_mask, x, expert_offsets, perm_slot,
                                       inv_perm, x_perm, counts, /*chunk=*/nullptr,
                                       /*status=*/nullptr,
                                       device_sm_count(), s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
