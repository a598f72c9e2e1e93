// Recombination of shared and routed expert outputs (Inkling layers page,
// InklingMoE.forward):
//   out[t] = sum_s y_shared[s*T + t] + sum_j y_routed[inv_perm[t*k + j]]
// in fp32, in that fixed order (shared s ascending, then choices j
// ascending), rounded once to the output dtype.  The rows are fp32, or fp16
// for MOE_BF16_F16DOWN layers (widened exactly before the sum).  The routing weights are
// already folded into the rows (inkling_swiglu multiplies silu(g)*u by them),
// so the sum is unweighted.  One block per token; 16-byte vector loads and
// stores along the hidden dim, coalesced across the block.  HBM-bound.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// acc[0..V) += V consecutive fp32 values (V = 8 or 4)
template <int V>
__device__ __forceinline__ void add_vec(float (&acc)[V], const float* p) {
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const float4 q = __ldcs(reinterpret_cast<const float4*>(p) + i);
    acc[4 * i + 0] += q.x;
    acc[4 * i + 1] += q.y;
    acc[4 * i + 2] += q.z;
    acc[4 * i + 3] += q.w;
  }
}

__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&acc)[8]) {
  uint4 q;
  q.x = pack_bf16x2(acc[0], acc[1]);
  q.y = pack_bf16x2(acc[2], acc[3]);
  q.z = pack_bf16x2(acc[4], acc[5]);
  q.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(p) = q;
}

__device__ __forceinline__ void store_vec(float* p, const float (&acc)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(acc[0], acc[1], acc[2], acc[3]);
}

// TY: output dtype; TR: expert row dtype (fp32)
template <typename TY, typename TR>
__global__ void __launch_bounds__(256)
    combine_kernel(const TR* __restrict__ y_routed, const TR* __restrict__ y_shared,
                   const int32_t* __restrict__ inv_perm, TY* __restrict__ out, int64_t T, int H,
                   int k, int S, int64_t rows_cap, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  constexpr int V = 16 / sizeof(TY);   // one 16-byte output store per vector
  __shared__ int s_rows[32];
  const int nv = H / V;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      int r = inv_perm[t * k + threadIdx.x];
      if (r >= rows_cap) {
        record_status(status, DEV_BAD_ROW);
        r = -1;
      }
      s_rows[threadIdx.x] = r;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.0f;
      for (int s = 0; s < S; ++s)
        add_vec(acc, y_shared + (static_cast<int64_t>(s) * T + t) * H + static_cast<int64_t>(v) * V);
      for (int j = 0; j < k; ++j) {
        const int r = s_rows[j];
        if (r >= 0) add_vec(acc, y_routed + static_cast<int64_t>(r) * H + static_cast<int64_t>(v) * V);
      }
      store_vec(out + t * H + static_cast<int64_t>(v) * V, acc);
    }
    __syncthreads();
  }
}

// Rows of TR (fp16, or fp32) into bf16 output: the same sums in the same
// order.  A vector is 8 values (one 16-byte load of fp16, two of fp32); each
// thread takes VPT vectors (VPT * blockDim vectors per pass; one pass for
// H <= VPT * 2048), so it keeps VPT * kRowBatch vectors of loads in flight,
// and the next token's row pointers are read while the current token is
// summed, so no dependent index load stalls the block between tokens.  The
// row batch (4 fp16 rows, 2 fp32 rows) keeps registers for two blocks an SM.
template <typename TR, int VPT>
__global__ void __launch_bounds__(256)
    combine_rows_kernel(const TR* __restrict__ y_routed, const TR* __restrict__ y_shared,
                        const int32_t* __restrict__ inv_perm, __nv_bfloat16* __restrict__ out,
                        int64_t T, int H, int k, int S, int64_t rows_cap, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  constexpr int kRowBatch = sizeof(TR) == 2 ? 4 : 2;
  constexpr int LPV = sizeof(TR) == 2 ? 1 : 2;   // 16-byte loads per vector of 8 values
  __shared__ const TR* s_src[2][32];   // a token's rows: S shared, then k routed (or null)
  const int nv = H / 8;
  const int n = S + k;
  auto row_of = [&](int64_t t, int i) -> const TR* {
    if (i < S) return y_shared + (static_cast<int64_t>(i) * T + t) * H;
    int r = inv_perm[t * k + (i - S)];
    if (r >= rows_cap) {
      record_status(status, DEV_BAD_ROW);
      r = -1;
    }
    return r >= 0 ? y_routed + static_cast<int64_t>(r) * H : nullptr;
  };
  int buf = 0;
  if (threadIdx.x < n && blockIdx.x < T) s_src[0][threadIdx.x] = row_of(blockIdx.x, threadIdx.x);
  __syncthreads();
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const int64_t tn = t + gridDim.x;
    const TR* nxt = nullptr;   // this thread's row of the next token
    if (threadIdx.x < n && tn < T) nxt = row_of(tn, threadIdx.x);
    for (int base = 0; base < nv; base += VPT * blockDim.x) {
      float acc[VPT][8];
#pragma unroll
      for (int j = 0; j < VPT; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][i] = 0.0f;
      for (int i0 = 0; i0 < n; i0 += kRowBatch) {
        uint4 q[kRowBatch][VPT][LPV];
#pragma unroll
        for (int u = 0; u < kRowBatch; ++u) {
          const TR* src = i0 + u < n ? s_src[buf][i0 + u] : nullptr;
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const int v = base + threadIdx.x + j * blockDim.x;
            if (src != nullptr && v < nv) {
#pragma unroll
              for (int l = 0; l < LPV; ++l)
                q[u][j][l] = __ldcs(reinterpret_cast<const uint4*>(src) + static_cast<int64_t>(v) * LPV + l);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kRowBatch; ++u) {
          if (i0 + u < n && s_src[buf][i0 + u] != nullptr) {   // rows in order; skipped rows add nothing
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
              if (sizeof(TR) == 2) {
                const uint32_t w[4] = {q[u][j][0].x, q[u][j][0].y, q[u][j][0].z, q[u][j][0].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
                  acc[j][2 * e] += f.x;
                  acc[j][2 * e + 1] += f.y;
                }
              } else {
#pragma unroll
                for (int l = 0; l < LPV; ++l) {
                  acc[j][4 * l + 0] += __uint_as_float(q[u][j][l].x);
                  acc[j][4 * l + 1] += __uint_as_float(q[u][j][l].y);
                  acc[j][4 * l + 2] += __uint_as_float(q[u][j][l].z);
                  acc[j][4 * l + 3] += __uint_as_float(q[u][j][l].w);
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = base + threadIdx.x + j * blockDim.x;
        if (v < nv) store_vec(out + t * H + static_cast<int64_t>(v) * 8, acc[j]);
      }
    }
    if (threadIdx.x < n) s_src[buf ^ 1][threadIdx.x] = nxt;
    buf ^= 1;
    __syncthreads();
  }
}

// bf16 output from rows of TR: vectors a thread sized to cover the row in
// one pass of 256 threads, at most 4 (longer rows take several passes)
template <typename TR>
cudaError_t launch_rows(unsigned grid, cudaStream_t stream, const TR* yr, const TR* ys,
                        const int32_t* inv_perm, __nv_bfloat16* o, const Layer& L, int64_t cap,
                        int32_t* status) {
  const int nv = L.H / 8;
  auto* kernel = nv <= 256   ? combine_rows_kernel<TR, 1>
                 : nv <= 512 ? combine_rows_kernel<TR, 2>
                 : nv <= 768 ? combine_rows_kernel<TR, 3>
                             : combine_rows_kernel<TR, 4>;
  return launch_chained(kernel, grid, 256, 0, stream, yr, ys, inv_perm, o, L.T, L.H, L.k, L.S,
                        cap, status);
}

}  // namespace

cudaError_t launch_combine(const Layer& L, const void* y_routed, const void* y_shared,
                           const int32_t* inv_perm, void* out, int32_t* status, int num_sms,
                           cudaStream_t stream) {
  const unsigned grid =
      static_cast<unsigned>(std::min<int64_t>(L.T, static_cast<int64_t>(num_sms) * 8));
  const int64_t cap = L.T * L.k;
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (L.dtype == MOE_BF16 && L.y_f16)
    return launch_rows(grid, stream, static_cast<const __half*>(y_routed),
                       static_cast<const __half*>(y_shared), inv_perm, o, L, cap, status);
  if (L.dtype == MOE_BF16)
    return launch_rows(grid, stream, static_cast<const float*>(y_routed),
                       static_cast<const float*>(y_shared), inv_perm, o, L, cap, status);
  return launch_chained(combine_kernel<float, float>, grid, 256, 0, stream,
                        static_cast<const float*>(y_routed), static_cast<const float*>(y_shared),
                        inv_perm, static_cast<float*>(out), L.T, L.H, L.k, L.S, cap, status);
}

}  // namespace moe
