// RMSNorm of the feed-forward block's input (InklingRMSNorm on the NeMo
// AutoModel Inkling "text" page; the decoder layer's post_attention_layernorm):
//   out[t, :] = x[t, :] / sqrt(mean_h x[t, h]^2 + eps) * weight
// rounded once to the input dtype.  The arithmetic is fp64: squares of bf16
// or fp32 values are exact in fp64, the row sum carries ~1e-16 relative
// error, and the row's 1/sqrt(mean + eps) is one correctly rounded fp64
// square root and division, so the rounded result is the exact value's
// rounding except within ~1e-16 of a tie.  (The page states fp32 variance
// accumulation; fp64 is at least that, and it makes the bf16 rounding, which
// decides the top-k selection downstream, reproducible.)  The rounding to
// bf16 is done here on the fp64 bit pattern, round to nearest with ties to
// even, in one step.
//
// Rows of up to 1024 vectors (bf16: H <= 8192; fp32: H <= 4096) run in
// rmsnorm_rows_kernel: a team of TPR threads (32..256, one to eight warps)
// per row, each thread holding up to four 16-byte vectors of its row in
// registers.  Every vector of the row is loaded at once (one HBM read per
// element, all of a row's loads in flight together, and the next row's
// issued before this row's reduction), each thread adds its
// squares into fp64 partials per element position, the warps reduce by a
// butterfly and the row's warps' sums are added in warp order through shared
// memory (a fixed order: the same sum on every run), and the thread scales
// and stores the vectors it holds.  Longer rows take the streamed kernel
// below.
//
// Streamed kernel: one warp per token row, 16-byte vectors along the row, streamed twice:
// pass 1 sums the squares, pass 2 re-reads the row (from L1: a few blocks
// per SM keep their rows there) and writes the result.  Both passes load
// their vectors in explicit batches (RMS_BATCH vectors a lane in registers
// before any is used), so each warp keeps RMS_BATCH x 512 bytes in flight,
// and pass 1 adds into one fp64 partial sum per element position of a
// vector (8 short chains instead of one long one); the partials are added in
// a fixed order, then across the warp by a butterfly, which leaves the same
// sum in every lane.  Each element is
// scaled by the row's 1/s, s = sqrt(mean + eps), computed once per row in
// fp64.  bf16 layers: x * weight is exact in fp32 (two 8-bit significands);
// y32 = (x * weight) * fp32(1/s) is within 2^-23 |y| (under 2 fp32 ulps) of
// the exact y, so when y32 is at least 4 ulps from a bf16 rounding tie it
// rounds like y, and it is rounded directly; otherwise (about 1 element in
// 8000) y is formed in fp64 and rounded from there.  fp32 layers multiply in
// fp64.  Against x / s * weight in fp64 the result differs only within
// ~1e-16 of a tie.  HBM-bound: 2 x dtype bytes per element.  `out` may alias
// `x` (a lane writes only vectors it has read).
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

#ifndef RMS_BATCH
#define RMS_BATCH 4
#endif
#ifndef RMS_BLOCKS_PER_SM
#define RMS_BLOCKS_PER_SM 4
#endif

struct Bf16Row {
  using Vec = uint4;                      // 8 bf16
  static constexpr int V = 8;
  // acc[i] += square of element i (squares of bf16 values are exact)
  __device__ static void sumsq(const Vec& q, double (&acc)[V]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xFFFF0000u);
      acc[2 * i] = fma(a, a, acc[2 * i]);
      acc[2 * i + 1] = fma(b, b, acc[2 * i + 1]);
    }
  }
  // acc[i & 1] += square of element i
  __device__ static void sumsq2(const Vec& q, double (&acc)[2]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xFFFF0000u);
      acc[0] = fma(a, a, acc[0]);
      acc[1] = fma(b, b, acc[1]);
    }
  }
  // bf16 bits of p * inv (p = x * weight, exact in fp32)
  __device__ static uint32_t one(float p, float inv32, double inv) {
    const float y32 = p * inv32;
    const uint32_t b = __float_as_uint(y32);
    const int from_tie = static_cast<int>(b & 0xFFFFu) - 0x8000;
    if ((from_tie >= -3 && from_tie <= 3) || fabsf(y32) < 0x1p-120f)
      return bf16_bits_rne(static_cast<double>(p) * inv);
    return (b + 0x8000u) >> 16;          // not a tie: round to nearest
  }
  __device__ static Vec scale(const Vec& q, const Vec& g, float inv32, double inv) {
    const uint32_t xw[4] = {q.x, q.y, q.z, q.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(xw[i] << 16) * __uint_as_float(gw[i] << 16);
      const float hi = __uint_as_float(xw[i] & 0xFFFF0000u) * __uint_as_float(gw[i] & 0xFFFF0000u);
      o[i] = one(lo, inv32, inv) | (one(hi, inv32, inv) << 16);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  }
};

struct F32Row {
  using Vec = float4;
  static constexpr int V = 4;
  // squares of fp32 values are exact in fp64
  __device__ static void sumsq(const Vec& q, double (&acc)[V]) {
    acc[0] = fma(static_cast<double>(q.x), q.x, acc[0]);
    acc[1] = fma(static_cast<double>(q.y), q.y, acc[1]);
    acc[2] = fma(static_cast<double>(q.z), q.z, acc[2]);
    acc[3] = fma(static_cast<double>(q.w), q.w, acc[3]);
  }
  __device__ static void sumsq2(const Vec& q, double (&acc)[2]) {
    acc[0] = fma(static_cast<double>(q.x), q.x, acc[0]);
    acc[1] = fma(static_cast<double>(q.y), q.y, acc[1]);
    acc[0] = fma(static_cast<double>(q.z), q.z, acc[0]);
    acc[1] = fma(static_cast<double>(q.w), q.w, acc[1]);
  }
  __device__ static Vec scale(const Vec& q, const Vec& g, float, double inv) {
    return make_float4(__double2float_rn(static_cast<double>(q.x) * g.x * inv),
                       __double2float_rn(static_cast<double>(q.y) * g.y * inv),
                       __double2float_rn(static_cast<double>(q.z) * g.z * inv),
                       __double2float_rn(static_cast<double>(q.w) * g.w * inv));
  }
};

template <typename R>
__global__ void __launch_bounds__(kThreads)
    rmsnorm_kernel(const void* x_, const void* __restrict__ w_, void* out_, int64_t T, int H,
                   double eps) {
  pdl_wait();
  pdl_trigger();
  using Vec = typename R::Vec;
  constexpr int B = RMS_BATCH;
  const Vec* x = static_cast<const Vec*>(x_);
  const Vec* w = static_cast<const Vec*>(w_);
  Vec* out = static_cast<Vec*>(out_);
  const int nv = H / R::V;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); t < T;
       t += warps) {
    const Vec* row = x + t * nv;
    Vec* orow = out + t * nv;
    double part[R::V];
#pragma unroll
    for (int i = 0; i < R::V; ++i) part[i] = 0.0;
    for (int v0 = lane; v0 < nv; v0 += 32 * B) {
      Vec buf[B];
#pragma unroll
      for (int j = 0; j < B; ++j)
        if (v0 + 32 * j < nv) buf[j] = row[v0 + 32 * j];
#pragma unroll
      for (int j = 0; j < B; ++j)
        if (v0 + 32 * j < nv) R::sumsq(buf[j], part);
    }
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < R::V; ++i) acc += part[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const double inv = 1.0 / sqrt(acc / H + eps);
    const float inv32 = __double2float_rn(inv);
    for (int v0 = lane; v0 < nv; v0 += 32 * B) {
      Vec buf[B], gw[B];
#pragma unroll
      for (int j = 0; j < B; ++j)
        if (v0 + 32 * j < nv) {
          buf[j] = row[v0 + 32 * j];
          gw[j] = w[v0 + 32 * j];
        }
#pragma unroll
      for (int j = 0; j < B; ++j)
        if (v0 + 32 * j < nv) orow[v0 + 32 * j] = R::scale(buf[j], gw[j], inv32, inv);
    }
  }
}

// Row-resident variant: TPR = 1 << tpr_log2 threads per row (32..256), each
// holding VPT vectors; 256 / TPR rows per block.  The loop over row groups
// is uniform across the block (every thread reaches every barrier).  The
// next row group's vectors are loaded before the current group's block
// reduction, so that each block keeps two rows' loads in flight.
template <typename R, int VPT>
__global__ void __launch_bounds__(kThreads, 4)
    rmsnorm_rows_kernel(const void* x_, const void* __restrict__ w_, void* out_, int64_t T, int H,
                        double eps, int tpr_log2) {
  pdl_wait();
  pdl_trigger();
  using Vec = typename R::Vec;
  __shared__ double s_part[kThreads / 32];
  const Vec* x = static_cast<const Vec*>(x_);
  const Vec* w = static_cast<const Vec*>(w_);
  Vec* out = static_cast<Vec*>(out_);
  const int nv = H / R::V;
  const int tpr = 1 << tpr_log2;
  const int rpb = kThreads >> tpr_log2;                  // rows per block
  const int r_in_b = threadIdx.x >> tpr_log2;
  const int t_in_r = threadIdx.x & (tpr - 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpr = tpr >> 5;                              // warps per row
  const int first_warp = r_in_b * wpr;
  const int64_t step = static_cast<int64_t>(gridDim.x) * rpb;
  auto load_row = [&](int64_t t, Vec (&buf)[VPT]) {
    if (t >= T) return;
    const Vec* row = x + t * nv;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = t_in_r + j * tpr;
      if (v < nv) buf[j] = row[v];
    }
  };
  Vec buf[VPT];
  int64_t base = static_cast<int64_t>(blockIdx.x) * rpb;
  load_row(base + r_in_b, buf);
  for (; base < T; base += step) {
    const int64_t t = base + r_in_b;
    const bool live = t < T;
    Vec nxt[VPT];
    load_row(base + step + r_in_b, nxt);                 // in flight during this row's reduction
    // two fp64 partial sums a thread (element positions even / odd), added
    // in a fixed order
    double part[2] = {0.0, 0.0};
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = t_in_r + j * tpr;
      if (live && v < nv) R::sumsq2(buf[j], part);
    }
    double acc = part[0] + part[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_part[warp] = acc;
    __syncthreads();
    double total = 0.0;
    for (int i = 0; i < wpr; ++i) total += s_part[first_warp + i];   // warp order
    __syncthreads();                                     // s_part free for the next rows
    if (live) {
      const double inv = 1.0 / sqrt(total / H + eps);
      const float inv32 = __double2float_rn(inv);
      Vec* orow = out + t * nv;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = t_in_r + j * tpr;
        if (v < nv) orow[v] = R::scale(buf[j], w[v], inv32, inv);
      }
    }
#pragma unroll
    for (int j = 0; j < VPT; ++j) buf[j] = nxt[j];
  }
}

template <typename R>
cudaError_t launch_rows(int64_t T, int H, double eps, const void* x, const void* weight,
                        void* out, int num_sms, cudaStream_t stream) {
  const int nv = H / R::V;
  // the fewest threads per row (32..256) that hold the row in at most 4
  // vectors a thread; fewer vectors a thread when the row allows it
  int tpr_log2 = 5;
  while ((1 << tpr_log2) * 4 < nv && tpr_log2 < 8) ++tpr_log2;
  const int tpr = 1 << tpr_log2;
  const int vpt = (nv + tpr - 1) / tpr;
  const int rpb = kThreads / tpr;
  const int64_t blocks = (T + rpb - 1) / rpb;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(blocks, static_cast<int64_t>(num_sms) * 4));
  auto* kernel = vpt == 1   ? rmsnorm_rows_kernel<R, 1>
                 : vpt == 2 ? rmsnorm_rows_kernel<R, 2>
                 : vpt == 3 ? rmsnorm_rows_kernel<R, 3>
                            : rmsnorm_rows_kernel<R, 4>;
  return launch_chained(kernel, grid, kThreads, 0, stream, x, weight, out, T, H, eps, tpr_log2);
}

}  // namespace

cudaError_t launch_rmsnorm(int64_t T, int H, int dtype, float eps, const void* x,
                           const void* weight, void* out, int num_sms, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  // rows of at most 1024 vectors: held in registers by a team of threads
  if (H / (dtype == MOE_BF16 ? Bf16Row::V : F32Row::V) <= 1024)
    return dtype == MOE_BF16 ? launch_rows<Bf16Row>(T, H, eps, x, weight, out, num_sms, stream)
                             : launch_rows<F32Row>(T, H, eps, x, weight, out, num_sms, stream);
  // longer rows: one warp per row, 8 rows per block, a few blocks per SM
  // (rows re-read from L1)
  const int64_t blocks = (T + kThreads / 32 - 1) / (kThreads / 32);
  const unsigned grid = static_cast<unsigned>(
      std::min<int64_t>(blocks, static_cast<int64_t>(num_sms) * RMS_BLOCKS_PER_SM));
  return launch_chained(dtype == MOE_BF16 ? rmsnorm_kernel<Bf16Row> : rmsnorm_kernel<F32Row>, grid,
                        kThreads, 0, stream, x, weight, out, T, H, static_cast<double>(eps));
}

}  // namespace moe
