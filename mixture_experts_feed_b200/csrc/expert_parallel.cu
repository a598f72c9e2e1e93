// Expert parallelism: the routed experts sharded over W ranks, one GPU each
// (Inkling layers page: GroupedExperts provides expert-parallel sharding, and
// the parallelizer shards InklingMoE.experts over the expert-parallel mesh).
//
// Rank r owns the routed experts [r*El, (r+1)*El), El = E / W, and keeps the
// router bank and the shared experts whole.  A step on rank r:
//   moe_route, moe_permute over its own tokens: rows ordered by global
//     expert, so the rows for rank d are one run, sub-ordered by expert;
//   moe_ep_dispatch_prep (this file): the routing weight of every permuted
//     row (it travels with the row) and the per-expert row counts;
//   the counts go to every rank (an all-to-all of E int32 a rank), then each
//     (destination, expert) run of rows and weights goes straight to its place
//     in the destination's expert-major buffer (grouped send/receive);
//   moe_expert_ffn over the received rows, already grouped by local expert
//     (perm_slot = NULL: row g's weight is the g-th received weight);
//   the output rows go back the same way into the sender's permuted order;
//   moe_shared_ffn over its own tokens, and moe_combine as on one GPU.
// The exchanges and their host-side bookkeeping are in the Python binding
// (mixture_experts_feed_b200/ep.py); every arithmetic step is a kernel.
#include <algorithm>

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "inkling_moe.h"
#include "internal.h"

namespace moe {
namespace {

// row_w[r] = topk_w[perm_slot[r]] for the R = offsets[E] permuted rows,
// counts[e] = offsets[e+1] - offsets[e].  A slot outside [0, slots) is
// recorded in the status word and its row gets weight 0.
__global__ void ep_dispatch_prep_kernel(const int32_t* __restrict__ offsets,
                                        const int32_t* __restrict__ perm_slot,
                                        const float* __restrict__ topk_w, int E, int64_t slots,
                                        float* __restrict__ row_w, int32_t* __restrict__ counts,
                                        int32_t* status) {
  int64_t R = offsets[E];
  if (R < 0 || R > slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, DEV_BAD_ROW);
    R = R < 0 ? 0 : slots;
  }
  const int64_t n = R > E ? R : E;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    if (i < E) counts[i] = offsets[i + 1] - offsets[i];
    if (i < R) {
      const int slot = perm_slot[i];
      if (slot >= 0 && slot < slots) {
        row_w[i] = topk_w[slot];
      } else {
        record_status(status, DEV_BAD_ROW);
        row_w[i] = 0.0f;
      }
    }
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_ep_dispatch_prep(const moe_layer_desc_t* desc,
                                             const int32_t* expert_offsets,
                                             const int32_t* perm_slot, const float* topk_w,
                                             float* row_w, int32_t* expert_counts, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  Layer L;
  const moe_status_t st = validate_desc(desc, &L);
  if (st != MOE_OK) return st;
  if (expert_offsets == nullptr || perm_slot == nullptr || topk_w == nullptr ||
      row_w == nullptr || expert_counts == nullptr || workspace == nullptr ||
      (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 || workspace_bytes < 256)
    return MOE_ERR_INVALID_ARG;
  const int64_t slots = L.T * L.k;
  const int64_t n = std::max<int64_t>(slots, L.E);
  const unsigned grid = static_cast<unsigned>(
      std::min<int64_t>(ceil_div(n, 256), static_cast<int64_t>(device_sm_count()) * 4));
  ep_dispatch_prep_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      expert_offsets, perm_slot, topk_w, L.E, slots, row_w, expert_counts,
      static_cast<int32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
