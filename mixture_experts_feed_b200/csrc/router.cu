// InklingGate on the GPU (Inkling layers page, InklingGate docstring and
// InklingCorrectionBias.forward).
//
// Kernels:
//   router_split_kernel   (bf16 layers) splits the fp32 gate bank exactly into
//                         three bf16 parts W = W0 + W1 + W2 (8 + 8 + 8
//                         significand bits), so that the logits can run on the
//                         tensor cores with every product exact in fp32
//                         (grouped_gemm_sm100.cu, kRouter).
//   router_logits_kernel  (fp32 layers) z[t, e] = sum_h x[t, h] * Wr[e, h] in
//                         fp32 FFMA, tiled 64 tokens x 64 rows x 32 K.
//   Both give fp32 logits for all E routed + S shared rows of the gate bank
//   (the gate runs in fp32: gate_precision=torch.float32).
//   router_sum_splits_kernel  (many K splits, few tokens) partial logits summed
//                         by eight threads a logit: eighths of the splits in
//                         order, then a fixed tree
//   router_topk_kernel    one warp per token: selection score
//                         sigmoid(z) + bias over the routed rows, k rounds of
//                         a warp-wide argmax (two warp reduction
//                         instructions a round: the largest score, then the
//                         lowest expert id holding it), then the weights.  The softmax over
//                         log-sigmoid(z) of [selected ++ shared] equals
//                         sigmoid(z_i) / sum sigmoid(z), which is what the
//                         kernel evaluates, times route_scale*global_scale.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int RL_BM = 64, RL_BN = 64, RL_BK = 32, RL_THREADS = 256;

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// Exact three-way bf16 split of fp32 values: each part is the round-to-
// nearest bf16 of what the previous parts left over; the residual after
// three parts is zero for every finite fp32 input of normal range.
__global__ void router_split_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ parts,
                                    int64_t n) {
  pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float v = w[i];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
    const float r0 = v - __bfloat162float(p0);
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r0);
    const float r1 = r0 - __bfloat162float(p1);
    parts[i] = p0;
    parts[n + i] = p1;
    parts[2 * n + i] = __float2bfloat16_rn(r1);
  }
}

template <typename TX>
__global__ void __launch_bounds__(RL_THREADS)
    router_logits_kernel(const TX* __restrict__ x, const float* __restrict__ w,
                         float* __restrict__ z, int64_t T, int H, int NE, int ld) {
  __shared__ __align__(16) float As[RL_BK][RL_BM + 4];
  __shared__ __align__(16) float Bs[RL_BK][RL_BN + 4];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * RL_BM;
  const int n0 = blockIdx.y * RL_BN;
  const int tx = tid & 15, ty = tid >> 4;
  const int lr = tid >> 2, lk = (tid & 3) * 8;
  const int64_t arow = m0 + lr;
  const int brow = n0 + lr;
  const bool a_ok = arow < T, b_ok = brow < NE;
  const TX* ap = x + (a_ok ? arow : 0) * H + lk;
  const float* bp = w + static_cast<int64_t>(b_ok ? brow : 0) * H + lk;

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < H; k0 += RL_BK) {
    float av[8], bv[8];
    if (a_ok) load8(ap + k0, av); else {
#pragma unroll
      for (int i = 0; i < 8; ++i) av[i] = 0.0f;
    }
    if (b_ok) load8(bp + k0, bv); else {
#pragma unroll
      for (int i = 0; i < 8; ++i) bv[i] = 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      As[lk + i][lr] = av[i];
      Bs[lk + i][lr] = bv[i];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < RL_BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float ar[4] = {a.x, a.y, a.z, a.w};
      const float br[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty * 4 + i;
    if (row >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (col < NE) z[row * ld + col] = acc[i][j];
    }
  }
}

__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

constexpr int TK_WARPS = 8;
// From this many K splits on, and below this many tokens (a top-k grid of
// few warps, each of which would read every split of its logits), a
// separate kernel sums the partial logits first.
constexpr int kSumSplitsFrom = 4;
constexpr int64_t kSumSplitsBelowT = 2048;

// Sum the K-split partial logits into split 0 (many splits, few tokens).
// Eight consecutive lanes of a warp hold one logit: lane q adds the splits
// [ks * q / 8, ks * (q + 1) / 8) in order, then the eight sums combine in a
// fixed tree (neighbours, then pairs, then fours), which every one of the
// eight lanes computes alike; lane 0 of the eight stores it.  Short chains
// over 8x the threads: the launch is latency-bound.
__global__ void router_sum_splits_kernel(float* __restrict__ z, int ld, int ksplit, int64_t T,
                                         int NE) {
  pdl_wait();
  pdl_trigger();
  const int64_t split = T * static_cast<int64_t>(ld);
  const int64_t total = T * static_cast<int64_t>(NE) * 8;   // eight threads a logit
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31, q = lane & 7;
  // whole warps iterate together (the shuffles below take all 32 lanes)
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
       base < total; base += stride) {
    const int64_t i = (base + lane) >> 3;                   // this lane's logit
    const bool live = base + lane < total;
    float* zt = z;
    float v = 0.0f;
    if (live) {
      const int64_t t = i / NE;
      zt = z + t * ld + (i - t * NE);
      for (int s2 = ksplit * q / 8; s2 < ksplit * (q + 1) / 8; ++s2) v += zt[s2 * split];
    }
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (live && q == 0) zt[0] = v;
  }
}

// PL: routed scores held per lane (E <= 32 * PL).
template <int PL>
__global__ void __launch_bounds__(TK_WARPS * 32)
    router_topk_kernel(const float* __restrict__ z, int ld, int ksplit,
                       const float* __restrict__ bias, int64_t T, int E, int k, int S, float scale,
                       float* __restrict__ topk_w, int32_t* __restrict__ topk_idx,
                       float* __restrict__ gamma) {
  __shared__ int s_chosen[TK_WARPS][32];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * TK_WARPS + warp;
  if (t >= T) return;
  const float* zt = z + t * ld;
  const int64_t split = T * static_cast<int64_t>(ld);
  // logit of row e: the K-split partial sums added in split order
  auto logit = [&](int e) {
    float v = zt[e];
    for (int s2 = 1; s2 < ksplit; ++s2) v += zt[s2 * split + e];
    return v;
  };

  // Selection scores as order-preserving unsigned keys (a larger score has a
  // larger key; -0 is taken as +0, a NaN score ranks with -inf, and a row
  // past E gets key 0, below every score), so that a warp-wide maximum is one
  // reduction instruction.
  uint32_t key[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      float v = sigmoidf_(logit(e)) + bias[e];
      if (isnan(v)) v = -INFINITY;   // a NaN score ranks last, never breaks the argmax
      if (v == 0.0f) v = 0.0f;
      const uint32_t u = __float_as_uint(v);
      key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    } else {
      key[i] = 0u;
    }
  }
  // k rounds: each lane offers its best remaining score (strict '>' keeps
  // the lowest id among its equal scores), the warp takes the largest, and
  // among the lanes offering it the lowest expert id.
  uint32_t taken = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u, bi = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      if (!((taken >> i) & 1u) && key[i] > bk) {
        bk = key[i];
        bi = static_cast<uint32_t>(lane + 32 * i);
      }
    }
    const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
    uint32_t win = __reduce_min_sync(0xffffffffu, bk == top ? bi : 0xffffffffu);
    if (win >= static_cast<uint32_t>(E)) win = 0;   // unreachable for k <= E; keeps every index in range
    if ((win & 31u) == static_cast<uint32_t>(lane)) taken |= 1u << (win >> 5);
    if (lane == 0) s_chosen[warp][j] = static_cast<int>(win);
  }
  __syncwarp();
  float sg = 0.0f;
  if (lane < k) sg = sigmoidf_(logit(s_chosen[warp][lane]));
  else if (lane < k + S) sg = sigmoidf_(logit(E + (lane - k)));
  float sum = sg;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
  const float wv = sg / sum * scale;
  if (lane < k) {
    topk_w[t * k + lane] = wv;
    topk_idx[t * k + lane] = s_chosen[warp][lane];
  } else if (lane < k + S) {
    gamma[t * S + (lane - k)] = wv;
  }
}

}  // namespace

cudaError_t launch_router_split(const Layer& L, const float* w_router, void* w_parts,
                                int num_sms, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(L.E + L.S) * L.H;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), num_sms * 8));
  return launch_chained(router_split_kernel, grid, 256, 0, stream, w_router,
                        static_cast<__nv_bfloat16*>(w_parts), n);
}

cudaError_t launch_router_logits(const Layer& L, const void* x, const float* w_router,
                                 float* logits, int ld, cudaStream_t stream) {
  const int NE = L.E + L.S;
  dim3 grid(static_cast<unsigned>(ceil_div(L.T, RL_BM)), static_cast<unsigned>(ceil_div(NE, RL_BN)));
  if (L.dtype == MOE_BF16)
    return launch_chained(router_logits_kernel<__nv_bfloat16>, grid, RL_THREADS, 0, stream,
                          static_cast<const __nv_bfloat16*>(x), w_router, logits, L.T, L.H, NE, ld);
  return launch_chained(router_logits_kernel<float>, grid, RL_THREADS, 0, stream,
                        static_cast<const float*>(x), w_router, logits, L.T, L.H, NE, ld);
}

int router_topk_launches(int ksplit, int64_t T) {
  return ksplit >= kSumSplitsFrom && T < kSumSplitsBelowT ? 2 : 1;
}

cudaError_t launch_router_topk(const Layer& L, const float* logits, int ld, int ksplit,
                               const float* corr_bias, float* topk_w, int32_t* topk_idx,
                               float* shared_gamma, cudaStream_t stream) {
  if (router_topk_launches(ksplit, L.T) == 2) {
    const int NE = L.E + L.S;
    const int64_t n = L.T * static_cast<int64_t>(NE) * 8;   // eight threads a logit
    const unsigned sgrid = static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 148 * 8));
    const cudaError_t e = launch_chained(router_sum_splits_kernel, sgrid, 256, 0, stream,
                                         const_cast<float*>(logits), ld, ksplit, L.T, NE);
    if (e != cudaSuccess) return e;
    ksplit = 1;
  }
  const unsigned grid = static_cast<unsigned>(ceil_div(L.T, TK_WARPS));
  const float scale = L.route_scale * L.global_scale;
  const int pl = static_cast<int>(ceil_div(L.E, 32));
#define MOE_TOPK(PLV)                                                                       \
  launch_chained(router_topk_kernel<PLV>, grid, TK_WARPS * 32, 0, stream, logits, ld, ksplit, \
                 corr_bias, L.T, L.E, L.k, L.S, scale, topk_w, topk_idx, shared_gamma)
  cudaError_t e;
  if (pl <= 1) e = MOE_TOPK(1);
  else if (pl <= 2) e = MOE_TOPK(2);
  else if (pl <= 4) e = MOE_TOPK(4);
  else if (pl <= 8) e = MOE_TOPK(8);
  else if (pl <= 16) e = MOE_TOPK(16);
  else e = MOE_TOPK(32);
#undef MOE_TOPK
  return e;
}

}  // namespace moe
