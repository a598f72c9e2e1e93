// The activated rows of a gate_up projection whose K was split (the dense
// layer with few tokens, Inkling layers page: InklingDenseMLP's fused
// interleaved gate_up_proj and inkling_swiglu): the K-split partial
// accumulators P[s][t][2I] (fp32, columns interleaved [g0, u0, g1, u1, ...])
// are added in split order, then
//   h[t][j] = w * silu(g) * u,   g = sum_s P[s][t][2j],  u = sum_s P[s][t][2j+1]
// with the same fp32 expression as the grouped GEMM's gate_up epilogue, and
// rounded to bf16, or to fp16 for fp16 down projections (a value past the
// fp16 range is recorded in the status word).  HBM-bound on small buffers
// (they mostly stay in L2).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// one thread per 4 consecutive h values of a row (8 partial columns)
__global__ void swiglu_partials_kernel(const float* __restrict__ part, int ksplit, int64_t T,
                                       int I, float w, int f16, uint16_t* __restrict__ h,
                                       int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int groups = I / 4;
  const int64_t n = T * groups;
  const int64_t split = T * static_cast<int64_t>(2 * I);
  bool ovf = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / groups;
    const int j0 = static_cast<int>(i - t * groups) * 4;
    const float* p = part + t * (2 * I) + 2 * j0;
    float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    for (int s = 1; s < ksplit; ++s) {
      const float4 c = *reinterpret_cast<const float4*>(p + s * split);
      const float4 d = *reinterpret_cast<const float4*>(p + s * split + 4);
      a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
      b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
    }
    const float g[4] = {a.x, a.z, b.x, b.z}, u[4] = {a.y, a.w, b.y, b.w};
    float v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = w * __fdividef(g[q], 1.0f + __expf(-g[q])) * u[q];
    uint2 o;
    if (f16) {
      o.x = pack_f16x2(v[0], v[1], ovf);
      o.y = pack_f16x2(v[2], v[3], ovf);
    } else {
      o.x = pack_bf16x2(v[0], v[1]);
      o.y = pack_bf16x2(v[2], v[3]);
    }
    *reinterpret_cast<uint2*>(h + t * I + j0) = o;
  }
  if (ovf) record_status(status, DEV_F16_OVERFLOW);
}

}  // namespace

cudaError_t launch_swiglu_partials(const float* part, int ksplit, int64_t T, int I, float w,
                                   bool f16, void* h, int32_t* status, int num_sms,
                                   cudaStream_t stream) {
  const int64_t n = T * (I / 4);
  const unsigned grid = static_cast<unsigned>(
      std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, 256), static_cast<int64_t>(num_sms) * 8)));
  return launch_chained(swiglu_partials_kernel, grid, 256, 0, stream, part, ksplit, T, I, w,
                        f16 ? 1 : 0, static_cast<uint16_t*>(h), status);
}

}  // namespace moe
