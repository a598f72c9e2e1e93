// Token permutation for grouped dispatch (Inkling layers page, InklingMoE:
// grouped routed experts; InklingMoE.forward: padded tokens are excluded from
// routed dispatch).
//
// Rows are the live (token t, choice j) pairs ordered by (expert, token).
// Four kernels, none of which lets thread timing decide an order:
//   perm_count    per-expert histogram (order-free atomics), -1 in inv_perm
//                 for padded slots and slots with an out-of-range expert id
//   perm_scan     exclusive scan of the counts -> expert_offsets[E+1]
//   perm_compact  one block per expert walks the tokens in order; a block
//                 scan of "rows this token gives expert e" places each row
//   gather_rows   x_perm[r] = x[perm_slot[r] / k], one warp per row,
//                 16-byte coalesced copies
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void perm_count_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                                  int64_t T, int k, int E, int32_t* __restrict__ counts,
                                  int32_t* __restrict__ inv_perm, int32_t* status) {
  extern __shared__ int s_hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < T; t += stride) {
    const bool padded = pad != nullptr && pad[t] != 0;
    for (int j = 0; j < k; ++j) {
      const int64_t slot = t * k + j;
      const int e = idx[slot];
      if (padded) {
        inv_perm[slot] = -1;
      } else if (e < 0 || e >= E) {
        record_status(status, DEV_BAD_EXPERT_ID);
        inv_perm[slot] = -1;
      } else {
        atomicAdd(&s_hist[e], 1);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    if (s_hist[i] != 0) atomicAdd(&counts[i], s_hist[i]);
}

// Exclusive scan of counts[0..E) by one block of 1024 threads (E <= 1024).
__global__ void __launch_bounds__(1024)
    perm_scan_kernel(const int32_t* __restrict__ counts, int E, int32_t* __restrict__ offsets) {
  __shared__ int s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int v = tid < E ? counts[tid] : 0;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += u;
    }
    s_warp[lane] = wi - w;   // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = s_warp[warp] + incl - v;
  if (tid < E) offsets[tid] = excl;
  if (tid == E - 1) offsets[E] = excl + v;
}

constexpr int COMPACT_THREADS = 1024;

__global__ void __launch_bounds__(COMPACT_THREADS)
    perm_compact_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                        int64_t T, int k, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm_slot, int32_t* __restrict__ inv_perm) {
  __shared__ int s_warp[32];
  __shared__ int s_total;
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int begin = offsets[e];
  if (offsets[e + 1] == begin) return;   // no rows for this expert
  int running = begin;
  for (int64_t t0 = 0; t0 < T; t0 += COMPACT_THREADS) {
    const int64_t t = t0 + tid;
    uint32_t jm = 0;   // choices j of token t that picked expert e
    if (t < T && !(pad != nullptr && pad[t] != 0)) {
      const int32_t* it = idx + t * k;
      for (int j = 0; j < k; ++j)
        if (it[j] == e) jm |= 1u << j;
    }
    const int c = __popc(jm);
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int w = s_warp[lane];
      int wi = w;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, wi, d);
        if (lane >= d) wi += u;
      }
      s_warp[lane] = wi - w;
      if (lane == 31) s_total = wi;
    }
    __syncthreads();
    int r = running + s_warp[warp] + incl - c;
    while (jm != 0) {
      const int j = __ffs(jm) - 1;
      jm &= jm - 1;
      const int64_t slot = t * k + j;
      perm_slot[r] = static_cast<int32_t>(slot);
      inv_perm[slot] = r;
      ++r;
    }
    running += s_total;
    __syncthreads();
  }
}

template <typename TX>
__global__ void gather_rows_kernel(const TX* __restrict__ x, const int32_t* __restrict__ perm_slot,
                                   const int32_t* __restrict__ offsets, int E, int k, int H,
                                   int64_t slots, TX* __restrict__ x_perm, int32_t* status) {
  const int R = offsets[E];
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int nvec = H * static_cast<int>(sizeof(TX)) / 16;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < R; r += warps) {
    const int slot = perm_slot[r];
    if (slot < 0 || slot >= slots) {
      if (lane == 0) record_status(status, DEV_BAD_ROW);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(slot / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + r * H);
    for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
  }
}

}  // namespace

cudaError_t launch_permute(const Layer& L, const int32_t* topk_idx, const uint8_t* padding_mask,
                           const void* x, int32_t* offsets, int32_t* perm_slot, int32_t* inv_perm,
                           void* x_perm, int32_t* counts, int32_t* status, int num_sms,
                           cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * L.E, stream);
  if (err != cudaSuccess) return err;
  const int threads = 256;
  const unsigned cgrid = static_cast<unsigned>(
      std::min<int64_t>(ceil_div(L.T, threads), static_cast<int64_t>(num_sms) * 4));
  perm_count_kernel<<<cgrid, threads, sizeof(int) * L.E, stream>>>(topk_idx, padding_mask, L.T, L.k,
                                                                   L.E, counts, inv_perm, status);
  perm_scan_kernel<<<1, 1024, 0, stream>>>(counts, L.E, offsets);
  perm_compact_kernel<<<L.E, COMPACT_THREADS, 0, stream>>>(topk_idx, padding_mask, L.T, L.k,
                                                           offsets, perm_slot, inv_perm);
  const int64_t slots = L.T * L.k;
  const unsigned ggrid = static_cast<unsigned>(
      std::min<int64_t>(ceil_div(slots, 8), static_cast<int64_t>(num_sms) * 8));
  if (L.dtype == MOE_BF16)
    gather_rows_kernel<__nv_bfloat16><<<ggrid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), perm_slot, offsets, L.E, L.k, L.H, slots,
        static_cast<__nv_bfloat16*>(x_perm), status);
  else
    gather_rows_kernel<float><<<ggrid, 256, 0, stream>>>(static_cast<const float*>(x), perm_slot,
                                                         offsets, L.E, L.k, L.H, slots,
                                                         static_cast<float*>(x_perm), status);
  return cudaGetLastError();
}

}  // namespace moe
