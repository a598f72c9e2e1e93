// Shared device helpers of the Inkling MoE kernels: status word, bounded
// waits, bf16 packing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "inkling_moe.h"

namespace moe {

// Device status word codes (first int32 of the workspace).  Sticky: the first
// kernel to record a problem wins.
enum DeviceCode : int32_t {
  DEV_OK = 0,
  DEV_BAD_EXPERT_ID = 0x101,   // topk_idx outside [0, E)
  DEV_BAD_ROW = 0x102,         // inv_perm / perm_slot outside its range
  DEV_F16_OVERFLOW = 0x103,    // an activated value or expert output beyond the fp16 range
  DEV_WAIT_TIMEOUT = 0x201,    // a pipeline wait ran past its time limit
};

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

template <typename T> struct Vec16;   // 16-byte vector of T
template <> struct Vec16<float> { static constexpr int N = 4; };
template <> struct Vec16<__nv_bfloat16> { static constexpr int N = 8; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two fp32 values rounded to nearest fp16; `overflow` is set when either
// rounds to an infinity (|v| at or beyond 65520) or is not finite: an fp16
// whose exponent field is all ones.  Branch-free (one per-halfword compare),
// since epilogues pack dozens of values between two tensor-memory loads.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi, bool& overflow) {
  const __half2 h = __floats2half2_rn(lo, hi);
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
  overflow |= __vcmpeq2(u & 0x7C007C00u, 0x7C007C00u) != 0u;
  return u;
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Programmatic dependent launch.  The layer's kernels are launched with
// programmatic stream serialisation (launch_chained): a kernel's CTAs may
// start while the previous kernel on the stream is still finishing, so the
// launch latency and the kernel's own setup overlap that kernel's tail.
// Until pdl_wait() a kernel touches no global memory other than its
// parameters (it initialises shared-memory barriers, allocates tensor
// memory, prefetches tensor maps); pdl_wait() returns once the previous grid
// has completed and its writes are visible, so every read of an earlier
// result and every global write (including writes to buffers an earlier
// kernel reads) comes after it.  pdl_trigger() lets the next kernel be
// scheduled once every CTA of this one has called it or exited.  Launched
// without the attribute, pdl_wait() returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
