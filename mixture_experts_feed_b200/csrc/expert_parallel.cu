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
//
// Over peer memory (NVLink between the GPUs of a node) the two exchanges are
// kernels of their own, each a gather fused with the transfer:
//   moe_ep_dispatch_p2p: every permuted row of this rank is read from x and
//     stored straight into its owner's receive buffer (ordinary stores for
//     this rank's own experts, peer stores for the others), with its weight;
//     no x_perm copy is made and no message is sent;
//   moe_ep_return_p2p: every received output row is stored straight into its
//     source's y rows, at the row's place in the source's permuted order.
// Each is followed, on the caller's side, by a barrier over the ranks (an
// all-reduce on the same stream) before anyone reads what was stored.  The
// kernels never wait on another rank: they only store.
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

// Row r's run: the largest i < n with starts[i] <= r (starts ascending,
// starts[0] == 0, r < starts[n]).
__device__ __forceinline__ int run_of(const int32_t* starts, int n, int64_t r) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (starts[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Copy one row of `bytes` (a multiple of 16) from src to dst, one warp,
// 16-byte vectors, four loads in flight per lane.
__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* dst, int nvec,
                                         int lane) {
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64),
                d = __ldg(src + v + 96);
    dst[v] = a;
    dst[v + 32] = b;
    dst[v + 64] = c;
    dst[v + 96] = d;
  }
  for (; v < nvec; v += 32) dst[v] = __ldg(src + v);
}

constexpr int kP2PThreads = 256;

// One warp per permuted row r < offsets[E]: expert e (offsets in shared
// memory, binary search), owner d = e / El, destination row
// dst_base[e] + (r - offsets[e]) of d's receive buffers; the row of x
// (token perm_slot[r] / k) goes to dst_x[d], its weight topk_w[perm_slot[r]]
// to dst_w[d].  Rows whose slot or destination falls outside its buffer are
// recorded in the status word and skipped.
__global__ void __launch_bounds__(kP2PThreads)
    ep_dispatch_p2p_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ perm_slot,
                           const int32_t* __restrict__ offsets, const float* __restrict__ topk_w,
                           const int32_t* __restrict__ dst_base, int E, int El, int k,
                           int row_bytes, int64_t slots, void* const* __restrict__ dst_x,
                           float* const* __restrict__ dst_w, int64_t dst_rows, int32_t* status) {
  extern __shared__ int32_t s_off[];   // offsets[0..E]
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = offsets[i];
  __syncthreads();
  int64_t R = s_off[E];
  if (R < 0 || R > slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, DEV_BAD_ROW);
    R = R < 0 ? 0 : slots;
  }
  const int lane = threadIdx.x & 31;
  const int nvec = row_bytes / 16;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R;
       r += warps) {
    const int e = run_of(s_off, E + 1, r);
    const int d = e / El;
    const int64_t row = static_cast<int64_t>(dst_base[e]) + (r - s_off[e]);
    const int slot = perm_slot[r];
    if (slot < 0 || slot >= slots || row < 0 || row >= dst_rows) {
      if (lane == 0) record_status(status, DEV_BAD_ROW);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(slot / k) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(dst_x[d]) + row * row_bytes);
    copy_row(src, dst, nvec, lane);
    if (lane == 0) dst_w[d][row] = topk_w[slot];
  }
  __threadfence_system();   // the stores reach the peers before the kernel is seen complete
}

// One warp per received row i < rows_in: its run (local expert el, source s)
// from run_start (El * W + 1 ascending entries, run el * W + s), destination
// row src_base[run] + (i - run_start[run]) of source s's rows dst_y[s].
__global__ void __launch_bounds__(kP2PThreads)
    ep_return_p2p_kernel(const uint8_t* __restrict__ y_in, int64_t rows_in,
                         const int32_t* __restrict__ run_start, const int32_t* __restrict__ src_base,
                         int runs, int W, int row_bytes, void* const* __restrict__ dst_y,
                         int64_t dst_rows, int32_t* status) {
  extern __shared__ int32_t s_run[];   // run_start[0..runs]
  for (int i = threadIdx.x; i <= runs; i += blockDim.x) s_run[i] = run_start[i];
  __syncthreads();
  if (s_run[runs] != rows_in) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, DEV_BAD_ROW);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int nvec = row_bytes / 16;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       i < rows_in; i += warps) {
    const int run = run_of(s_run, runs + 1, i);
    const int s = run % W;
    const int64_t row = static_cast<int64_t>(src_base[run]) + (i - s_run[run]);
    if (row < 0 || row >= dst_rows) {
      if (lane == 0) record_status(status, DEV_BAD_ROW);
      continue;
    }
    copy_row(reinterpret_cast<const uint4*>(y_in + i * row_bytes),
             reinterpret_cast<uint4*>(static_cast<uint8_t*>(dst_y[s]) + row * row_bytes), nvec,
             lane);
  }
  __threadfence_system();
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace {

bool ws_ok(const void* workspace, size_t bytes) {
  return workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255) == 0 && bytes >= 256;
}

unsigned p2p_grid(int64_t rows) {
  const int64_t warps = kP2PThreads / 32;
  return static_cast<unsigned>(std::max<int64_t>(
      1, std::min<int64_t>(ceil_div(rows, warps), static_cast<int64_t>(device_sm_count()) * 8)));
}

}  // namespace

extern "C" moe_status_t moe_ep_dispatch_p2p(const moe_layer_desc_t* desc, const void* x,
                                            const float* topk_w, const int32_t* perm_slot,
                                            const int32_t* expert_offsets, const int32_t* dst_base,
                                            int32_t n_ranks, void* const* dst_x,
                                            float* const* dst_w, int64_t dst_rows,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  Layer L;
  const moe_status_t st = validate_desc(desc, &L);
  if (st != MOE_OK) return st;
  if (n_ranks < 1 || L.E % n_ranks != 0 || dst_rows < 0) return MOE_ERR_INVALID_ARG;
  if (x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15) != 0 || topk_w == nullptr ||
      perm_slot == nullptr || expert_offsets == nullptr || dst_base == nullptr ||
      dst_x == nullptr || dst_w == nullptr || !ws_ok(workspace, workspace_bytes))
    return MOE_ERR_INVALID_ARG;
  if (L.T == 0) return MOE_OK;
  const int elt = L.dtype == MOE_BF16 ? 2 : 4;
  const int64_t slots = L.T * L.k;
  ep_dispatch_p2p_kernel<<<p2p_grid(slots), kP2PThreads, sizeof(int32_t) * (L.E + 1),
                           static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(x), perm_slot, expert_offsets, topk_w, dst_base, L.E,
      L.E / n_ranks, L.k, L.H * elt, slots, dst_x, dst_w, dst_rows,
      static_cast<int32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_ep_return_p2p(const moe_layer_desc_t* desc, const void* y_in,
                                          int64_t rows_in, const int32_t* run_start,
                                          const int32_t* src_base, int32_t n_ranks,
                                          void* const* dst_y, int64_t dst_rows, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  Layer L;
  const moe_status_t st = validate_desc(desc, &L);
  if (st != MOE_OK) return st;
  if (n_ranks < 1 || L.E % n_ranks != 0 || rows_in < 0 || dst_rows < 0 ||
      rows_in >= (int64_t{1} << 31))
    return MOE_ERR_INVALID_ARG;
  if ((rows_in > 0 && (y_in == nullptr || (reinterpret_cast<uintptr_t>(y_in) & 15) != 0)) ||
      run_start == nullptr || src_base == nullptr || dst_y == nullptr ||
      !ws_ok(workspace, workspace_bytes))
    return MOE_ERR_INVALID_ARG;
  if (rows_in == 0) return MOE_OK;
  // the expert output rows: fp16 for MOE_BF16_F16DOWN layers, else fp32
  const int elt = L.y_f16 ? 2 : 4;
  const int runs = L.E;   // El local experts x W sources
  ep_return_p2p_kernel<<<p2p_grid(rows_in), kP2PThreads, sizeof(int32_t) * (runs + 1),
                         static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(y_in), rows_in, run_start, src_base, runs, n_ranks, L.H * elt,
      dst_y, dst_rows, static_cast<int32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

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
