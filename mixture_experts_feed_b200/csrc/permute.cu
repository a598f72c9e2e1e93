// Token permutation for grouped dispatch (Inkling layers page, InklingMoE:
// grouped routed experts; InklingMoE.forward: padded tokens are excluded from
// routed dispatch).
//
// Rows are the live (token t, choice j) pairs ordered by (expert, token),
// i.e. by (expert, slot) with slot = t * k + j.  None of the kernels lets
// thread timing decide an order.  With a workspace:
//   perm_chunk_count  per chunk of slots, per-expert counts (block
//                     histogram), added into the totals; -1 in inv_perm for
//                     padded slots and slots with an out-of-range expert id
//   perm_chunk_scan   one block per expert: expert_offsets[e] (the totals
//                     of the experts before e), then the expert's running
//                     sum over the chunks: the first row of (expert, chunk)
//   perm_scatter      per chunk, 32 consecutive slots a warp: a slot's rank
//                     among earlier slots of its expert is its rank in its
//                     warp's match group plus the earlier warps' and
//                     iterations' counts
//   perm_one_chunk    at most 256 slots (few tokens): the three steps above
//                     for the one chunk in a single block of 256 threads
//                     (a slot a thread), with the same order
// Without one (moe_permute_noalloc): perm_count (totals only), perm_scan,
// and perm_compact: one block per expert walks the tokens in order.
//   gather_rows   x_perm[r] = x[perm_slot[r] / k], one warp per row,
//                 16-byte coalesced copies; skipped when x_perm is null (the
//                 gate_up GEMM then gathers the rows of x itself)
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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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

// Exclusive block scan of one int per thread (256 threads); s_warp holds 8.
__device__ __forceinline__ int block_excl_scan_256(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int t = s_warp[w];
    if (w < warp) before += t;
    total += t;
  }
  __syncthreads();
  return before + incl - v;
}

// Block e (of E blocks, 256 threads): offsets[e] = sum of the totals of the
// experts before e (offsets[E] from the last block), then chunk[e][c], the
// count of expert e in chunk c, becomes the first row of (expert e, chunk c):
// offsets[e] plus the exclusive scan over the chunks.
__global__ void __launch_bounds__(256)
    perm_chunk_scan_kernel(const int32_t* __restrict__ counts, int E, int n_chunks,
                           int32_t* __restrict__ offsets, int32_t* __restrict__ chunk) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_warp[8];
  const int e = blockIdx.x;
  int part = 0;
  for (int i = threadIdx.x; i < e; i += blockDim.x) part += counts[i];
  int excl_total = 0;
  (void)block_excl_scan_256(part, s_warp, excl_total);   // excl_total = sum over experts < e
  if (threadIdx.x == 0) {
    offsets[e] = excl_total;
    if (e == E - 1) offsets[E] = excl_total + counts[e];
  }
  // each thread takes a contiguous run of `per` chunks (n_chunks <= 2048)
  int32_t* row = chunk + static_cast<int64_t>(e) * n_chunks;
  const int per = (n_chunks + 255) / 256;
  const int c0 = threadIdx.x * per;
  int v[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = (i < per && c0 + i < n_chunks) ? row[c0 + i] : 0;
    sum += v[i];
  }
  int unused = 0;
  int run = excl_total + block_excl_scan_256(sum, s_warp, unused);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < per && c0 + i < n_chunks) row[c0 + i] = run;
    run += v[i];
  }
}

// Per chunk of `cs` slots: counts per expert (block histogram), written to
// chunk[e][c] and added into the totals.
__global__ void __launch_bounds__(256)
    perm_chunk_count_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                            int64_t slots, int k, int E, int64_t cs,
                            int32_t* __restrict__ counts, int32_t* __restrict__ chunk,
                            int32_t* __restrict__ inv_perm, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  const int64_t c = blockIdx.x;
  const int64_t end = min(slots, (c + 1) * cs);
  for (int64_t sl = c * cs + threadIdx.x; sl < end; sl += blockDim.x) {
    const bool padded = pad != nullptr && pad[sl / k] != 0;
    const int e = idx[sl];
    if (padded) {
      inv_perm[sl] = -1;
    } else if (e < 0 || e >= E) {
      record_status(status, DEV_BAD_EXPERT_ID);
      inv_perm[sl] = -1;
    } else {
      atomicAdd(&s_hist[e], 1);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    const int n = s_hist[i];
    chunk[static_cast<int64_t>(i) * gridDim.x + c] = n;
    if (n != 0) atomicAdd(&counts[i], n);
  }
}

// Per chunk: slot s goes to row chunk[e][c] + (earlier slots of expert e in
// this chunk).  Slots are taken 256 at a time in order; inside a warp the
// rank is the slot's position in its match group (lanes with the same
// expert), to which the earlier warps' counts (s_cnt) add; s_base[e] starts
// at chunk[e][c] and moves past each iteration's rows of expert e.  s_cnt is
// kept zero between iterations.
__global__ void __launch_bounds__(256)
    perm_scatter_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                        int64_t slots, int k, int E, int64_t cs,
                        const int32_t* __restrict__ chunk, int32_t* __restrict__ perm_slot,
                        int32_t* __restrict__ inv_perm, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;              // [8 warps][E]
  int* s_base = s_mem + 8 * E;     // [E]
  const int64_t c = blockIdx.x;
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) s_cnt[i] = 0;
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_base[i] = chunk[static_cast<int64_t>(i) * gridDim.x + c];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int64_t begin = c * cs, end = min(slots, begin + cs);
  for (int64_t s0 = begin; s0 < end; s0 += blockDim.x) {
    const int64_t sl = s0 + threadIdx.x;
    int e = -1;
    if (sl < end && !(pad != nullptr && pad[sl / k] != 0)) {
      const int v = idx[sl];
      if (v >= 0 && v < E) e = v;
    }
    const uint32_t grp = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(grp & lt);
    const int n = __popc(grp);
    if (e >= 0 && rank == 0) s_cnt[warp * E + e] = n;
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += s_cnt[w * E + e];
      const int64_t pos = static_cast<int64_t>(s_base[e]) + before + rank;
      if (pos >= 0 && pos < slots) {
        perm_slot[pos] = static_cast<int32_t>(sl);
        inv_perm[sl] = static_cast<int32_t>(pos);
      } else {
        record_status(status, DEV_BAD_ROW);
      }
    }
    __syncthreads();
    if (e >= 0 && rank == 0) {
      atomicAdd(&s_base[e], n);   // leaders of several warps: integer sum, any order
      s_cnt[warp * E + e] = 0;
    }
    __syncthreads();
  }
}

// At most 256 slots: counts, offsets and the stable scatter in one block
// (thread i holds slot i), in the order of the chunked kernels: a slot's row
// is its expert's first row plus the earlier warps' slots of that expert
// plus its rank in its warp's match group.
__global__ void __launch_bounds__(256)
    perm_one_chunk_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                          int64_t slots, int k, int E, int32_t* __restrict__ offsets,
                          int32_t* __restrict__ perm_slot, int32_t* __restrict__ inv_perm,
                          int32_t* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;             // [8 warps][E]
  int* s_base = s_mem + 8 * E;    // [E]: the counts, then each expert's first row
  __shared__ int s_warp[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < 9 * E; i += blockDim.x) s_mem[i] = 0;
  __syncthreads();
  int e = -1;   // this thread's slot's expert, or -1
  if (tid < slots) {
    const bool padded = pad != nullptr && pad[tid / k] != 0;
    const int v = idx[tid];
    if (padded) {
      inv_perm[tid] = -1;
    } else if (v < 0 || v >= E) {
      record_status(status, DEV_BAD_EXPERT_ID);
      inv_perm[tid] = -1;
    } else {
      e = v;
    }
  }
  if (e >= 0) atomicAdd(&s_base[e], 1);
  __syncthreads();
  // exclusive scan of the counts: thread t takes experts [t * per, t * per + per)
  const int per = (E + 255) / 256;   // at most 4 (E <= 1024)
  int c[4];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ee = tid * per + i;
    c[i] = (i < per && ee < E) ? s_base[ee] : 0;
    sum += c[i];
  }
  int total = 0;
  int run = block_excl_scan_256(sum, s_warp, total);   // its barriers order the reads above
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ee = tid * per + i;
    if (i < per && ee < E) {
      s_base[ee] = run;
      offsets[ee] = run;
    }
    run += c[i];
  }
  if (tid == 0) offsets[E] = total;
  const uint32_t grp = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(grp & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) s_cnt[warp * E + e] = __popc(grp);
  __syncthreads();
  if (e >= 0) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_cnt[w * E + e];
    const int64_t pos = static_cast<int64_t>(s_base[e]) + before + rank;
    if (pos >= 0 && pos < slots) {
      perm_slot[pos] = tid;
      inv_perm[tid] = static_cast<int32_t>(pos);
    } else {
      record_status(status, DEV_BAD_ROW);
    }
  }
}

constexpr int COMPACT_THREADS = 1024;

__global__ void __launch_bounds__(COMPACT_THREADS)
    perm_compact_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ pad,
                        int64_t T, int k, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm_slot, int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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
    // eight 16-byte loads in flight per lane before their stores; the
    // stores are marked evict-first (streaming), so that the copy, k times
    // the size of x, does not push the rows of x out of L2 before their
    // other k - 1 reads
    constexpr int U = 8;
    int v = lane;
    for (; v + 32 * (U - 1) < nvec; v += 32 * U) {
      uint4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u) t[u] = __ldg(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u) __stcs(dst + v + 32 * u, t[u]);
    }
    for (; v < nvec; v += 32) __stcs(dst + v, __ldg(src + v));
  }
}

}  // namespace

int64_t permute_chunk_slots(int64_t slots) {
  // 256 slots a chunk, more when that would exceed 2048 chunks
  const int64_t per = ceil_div(slots, int64_t{2048});
  return std::max<int64_t>(256, ceil_div(per, int64_t{256}) * 256);
}

int64_t permute_chunks(int64_t slots) {
  return slots == 0 ? 0 : ceil_div(slots, permute_chunk_slots(slots));
}

int permute_kernel_count(int64_t slots, bool workspace) {
  return workspace && slots <= kOneChunkSlots ? 2 : 4;   // with the row gather
}

cudaError_t launch_permute(const Layer& L, const int32_t* topk_idx, const uint8_t* padding_mask,
                           const void* x, int32_t* offsets, int32_t* perm_slot, int32_t* inv_perm,
                           void* x_perm, int32_t* counts, int32_t* chunk, int32_t* status,
                           int num_sms, cudaStream_t stream) {
  const int64_t slots = L.T * L.k;
  cudaError_t err = cudaSuccess;
  if (chunk != nullptr && slots <= kOneChunkSlots) {
    err = launch_chained(perm_one_chunk_kernel, 1, 256, sizeof(int) * 9 * L.E, stream, topk_idx,
                         padding_mask, slots, L.k, L.E, offsets, perm_slot, inv_perm, status);
  } else {
    err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * L.E, stream);
  }
  if (err != cudaSuccess) return err;
  if (chunk != nullptr && slots <= kOneChunkSlots) {
    // counted, scanned and scattered above
  } else if (chunk != nullptr) {
    const int64_t cs = permute_chunk_slots(slots);
    const int nc = static_cast<int>(permute_chunks(slots));
    err = launch_chained(perm_chunk_count_kernel, nc, 256, sizeof(int) * L.E, stream, topk_idx,
                         padding_mask, slots, L.k, L.E, cs, counts, chunk, inv_perm, status);
    if (err == cudaSuccess)
      err = launch_chained(perm_chunk_scan_kernel, L.E, 256, 0, stream, counts, L.E, nc, offsets,
                           chunk);
    if (err == cudaSuccess)
      err = launch_chained(perm_scatter_kernel, nc, 256, sizeof(int) * 9 * L.E, stream, topk_idx,
                           padding_mask, slots, L.k, L.E, cs, chunk, perm_slot, inv_perm, status);
  } else {
    const int threads = 256;
    const unsigned cgrid = static_cast<unsigned>(
        std::min<int64_t>(ceil_div(L.T, threads), static_cast<int64_t>(num_sms) * 4));
    err = launch_chained(perm_count_kernel, cgrid, threads, sizeof(int) * L.E, stream, topk_idx,
                         padding_mask, L.T, L.k, L.E, counts, inv_perm, status);
    if (err == cudaSuccess)
      err = launch_chained(perm_scan_kernel, 1, 1024, 0, stream, counts, L.E, offsets);
    if (err == cudaSuccess)
      err = launch_chained(perm_compact_kernel, L.E, COMPACT_THREADS, 0, stream, topk_idx,
                           padding_mask, L.T, L.k, offsets, perm_slot, inv_perm);
  }
  if (err != cudaSuccess || x_perm == nullptr) return err;   // x_perm null: the consumer gathers
  const unsigned ggrid = static_cast<unsigned>(
      std::min<int64_t>(ceil_div(slots, 8), static_cast<int64_t>(num_sms) * 8));
  if (L.dtype == MOE_BF16)
    return launch_chained(gather_rows_kernel<__nv_bfloat16>, ggrid, 256, 0, stream,
                          static_cast<const __nv_bfloat16*>(x), perm_slot, offsets, L.E, L.k, L.H,
                          slots, static_cast<__nv_bfloat16*>(x_perm), status);
  return launch_chained(gather_rows_kernel<float>, ggrid, 256, 0, stream,
                        static_cast<const float*>(x), perm_slot, offsets, L.E, L.k, L.H, slots,
                        static_cast<float*>(x_perm), status);
}

}  // namespace moe
