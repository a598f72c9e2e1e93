// One-time preparation of the down projections' weights for MOE_BF16_F16DOWN
// layers: the checkpoint's bf16 values rounded to nearest fp16.  A bf16 value
// has 8 significant bits and an fp16 normal value 11, so every bf16 value
// with magnitude in [2^-14, 65504], and zero, converts exactly; below 2^-14
// fp16 keeps bits down to 2^-24 (its subnormal spacing), so values from
// 2^-17 up convert exactly and smaller ones change by at most 2^-25.  A value
// beyond 65504 in magnitude (or a NaN) has no fp16 counterpart: each such
// element adds one to an optional device counter, so that the caller can
// refuse the copy.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "inkling_moe.h"
#include "internal.h"

namespace moe {
namespace {

__global__ void bf16_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                   int64_t nvec, int32_t* nonfinite) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int bad = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    const uint4 q = src[i];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      const __half2 h = __floats2half2_rn(lo, hi);
      if (__hisinf(h.x) || __hisnan(h.x)) ++bad;
      if (__hisinf(h.y) || __hisnan(h.y)) ++bad;
      o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (nonfinite != nullptr && bad != 0) atomicAdd(nonfinite, bad);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_convert_bf16_to_f16(int64_t n, const void* src, void* dst,
                                                int32_t* nonfinite, void* stream) {
  if (n < 0 || n % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (src == nullptr || dst == nullptr || (reinterpret_cast<uintptr_t>(src) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(dst) & 15) != 0)
    return MOE_ERR_INVALID_ARG;
  const int64_t nvec = n / 8;
  const unsigned grid = static_cast<unsigned>(
      std::min<int64_t>(ceil_div(nvec, 256), static_cast<int64_t>(device_sm_count()) * 8));
  bf16_to_f16_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), nvec, nonfinite);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
