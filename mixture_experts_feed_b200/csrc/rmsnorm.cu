// RMSNorm of the feed-forward block's input (InklingRMSNorm on the NeMo
// AutoModel Inkling "text" page; the decoder layer's post_attention_layernorm):
//   out[t, :] = x[t, :] / sqrt(mean_h x[t, h]^2 + eps) * weight
// rounded once to the input dtype.  The arithmetic is fp64: squares of bf16
// or fp32 values are exact in fp64, the row sum carries ~1e-16 relative
// error, and fp64 square root and division are correctly rounded, so the
// rounded result is the exact value's rounding except within ~1e-16 of a
// tie.  (The page states fp32 variance accumulation; fp64 is at least that,
// and it makes the bf16 rounding, which decides the top-k selection
// downstream, reproducible.)  The rounding to bf16 is done here on the fp64
// bit pattern, round to nearest with ties to even, in one step.
//
// One block of 256 threads per token row, 16-byte vectors along the row:
// pass 1 sums the squares (warp shuffles, then the 8 warp sums in a fixed
// order), pass 2 re-reads the row (L1/L2) and writes the result.  HBM-bound:
// 2 x dtype bytes per element.  `out` may alias `x` (each thread reads a
// vector in pass 2 before it writes the same vector).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

// Round a double to the nearest bf16 (ties to even); returns the bf16 bits.
__device__ __forceinline__ uint16_t bf16_bits_rne(double y) {
  double r;
  if (fabs(y) < 0x1p-126) {
    // bf16 subnormal range: spacing 2^-133; rint rounds ties to even
    r = rint(y * 0x1p133) * 0x1p-133;
  } else {
    // keep 7 fraction bits: carry when the 45 dropped bits exceed half, or
    // equal half with an odd kept last bit
    unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(y));
    const unsigned long long lsb = (b >> 45) & 1ull;
    b = (b + 0xFFFFFFFFFFFull + lsb) & ~0x1FFFFFFFFFFFull;
    r = __longlong_as_double(static_cast<long long>(b));
  }
  // r is a bf16 value (or out of range: the float conversion saturates to inf)
  return static_cast<uint16_t>(__float_as_uint(__double2float_rn(r)) >> 16);
}

struct Bf16Row {
  using Vec = uint4;                      // 8 bf16
  static constexpr int V = 8;
  __device__ static void unpack(const Vec& q, double (&d)[V]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      d[2 * i] = static_cast<double>(__uint_as_float(w[i] << 16));
      d[2 * i + 1] = static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
    }
  }
  __device__ static Vec pack(const double (&y)[V]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(bf16_bits_rne(y[2 * i])) |
             (static_cast<uint32_t>(bf16_bits_rne(y[2 * i + 1])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

struct F32Row {
  using Vec = float4;
  static constexpr int V = 4;
  __device__ static void unpack(const Vec& q, double (&d)[V]) {
    d[0] = q.x; d[1] = q.y; d[2] = q.z; d[3] = q.w;
  }
  __device__ static Vec pack(const double (&y)[V]) {
    return make_float4(__double2float_rn(y[0]), __double2float_rn(y[1]),
                       __double2float_rn(y[2]), __double2float_rn(y[3]));
  }
};

template <typename R>
__global__ void __launch_bounds__(kThreads)
    rmsnorm_kernel(const void* __restrict__ x_, const void* __restrict__ w_, void* out_, int64_t T,
                   int H, double eps) {
  using Vec = typename R::Vec;
  const Vec* x = static_cast<const Vec*>(x_);
  const Vec* w = static_cast<const Vec*>(w_);
  Vec* out = static_cast<Vec*>(out_);
  const int nv = H / R::V;
  __shared__ double s_warp[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const Vec* row = x + t * nv;
    double acc = 0.0;
    for (int v = threadIdx.x; v < nv; v += kThreads) {
      double d[R::V];
      R::unpack(row[v], d);
#pragma unroll
      for (int i = 0; i < R::V; ++i) acc = fma(d[i], d[i], acc);   // d*d exact
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_warp[warp] = acc;
    __syncthreads();
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) ss += s_warp[i];      // same order in every thread
    const double s = sqrt(ss / H + eps);
    for (int v = threadIdx.x; v < nv; v += kThreads) {
      double d[R::V], g[R::V], y[R::V];
      R::unpack(row[v], d);
      R::unpack(w[v], g);
#pragma unroll
      for (int i = 0; i < R::V; ++i) y[i] = d[i] / s * g[i];
      out[t * nv + v] = R::pack(y);
    }
    __syncthreads();   // s_warp is rewritten for the next row
  }
}

}  // namespace

cudaError_t launch_rmsnorm(int64_t T, int H, int dtype, float eps, const void* x,
                           const void* weight, void* out, int num_sms, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(T, static_cast<int64_t>(num_sms) * 8));
  if (dtype == MOE_BF16)
    rmsnorm_kernel<Bf16Row><<<grid, kThreads, 0, stream>>>(x, weight, out, T, H, eps);
  else
    rmsnorm_kernel<F32Row><<<grid, kThreads, 0, stream>>>(x, weight, out, T, H, eps);
  return cudaGetLastError();
}

}  // namespace moe
