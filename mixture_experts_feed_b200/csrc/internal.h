// Launch functions behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "inkling_moe.h"

namespace moe {

struct Layer {
  int64_t T;
  int H, E, k, S, I;
  int dtype;   // activations: MOE_F32 / MOE_BF16
  float route_scale, global_scale;
  // MOE_BF16_F16DOWN layers: the down projections' weights are fp16 and the
  // activated rows h are rounded to fp16 (dtype is MOE_BF16)
  bool down_f16 = false;
  // the expert output rows y_routed / y_shared are fp16 (MOE_BF16_F16DOWN MoE
  // layers); else fp32.  The dense layer keeps fp32 rows (its K-split partials).
  bool y_f16 = false;
};

// moe_api.cu: SM count of the current device (cached per device), and the
// host-side check of a layer description (fills `L` when it returns MOE_OK).
int device_sm_count();
moe_status_t validate_desc(const moe_layer_desc_t* d, Layer* L);

// router.cu (logits row stride `ld` = E+S rounded up to 32)
cudaError_t launch_router_split(const Layer& L, const float* w_router, void* w_parts,
                                int num_sms, cudaStream_t stream);
cudaError_t launch_router_logits(const Layer& L, const void* x, const float* w_router,
                                 float* logits, int ld, cudaStream_t stream);
// kernels launch_router_topk launches for this K-split count (1 or 2)
int router_topk_launches(int ksplit, int64_t T);
cudaError_t launch_router_topk(const Layer& L, const float* logits, int ld, int ksplit,
                               const float* corr_bias,
                               float* topk_w, int32_t* topk_idx, float* shared_gamma,
                               cudaStream_t stream);

// permute.cu
cudaError_t launch_permute(const Layer& L, const int32_t* topk_idx, const uint8_t* padding_mask,
                           const void* x, int32_t* offsets, int32_t* perm_slot, int32_t* inv_perm,
                           void* x_perm, int32_t* counts, int32_t* chunk, int32_t* status,
                           int num_sms, cudaStream_t stream);
// Chunks of slots the workspace path splits T*k slots into (at most 2048),
// and the slots per chunk; `chunk` holds E * permute_chunks(T*k) int32.
// chunk == nullptr selects the workspace-free path (one block per expert).
int64_t permute_chunk_slots(int64_t slots);
int64_t permute_chunks(int64_t slots);
// With a workspace and at most this many slots one kernel counts, scans and
// scatters; the kernels launch_permute launches, the row gather included.
constexpr int64_t kOneChunkSlots = 256;
int permute_kernel_count(int64_t slots, bool workspace);

// The workspace's status region: its first 256 bytes.  Byte 0 holds the
// sticky device status word; bytes kTileCounterOffset .. +7 hold the tile
// counters of the gate_up pair launch's dynamic schedule (two int32: one for
// a call with routed groups, one for a call of shared groups alone), which
// each call zeroes on its stream before its launches.
constexpr size_t kStatusBytes = 256;
constexpr size_t kTileCounterOffset = 64;

// grouped_gemm_sm100.cu (bf16, tcgen05)
// Tile shape choices of one expert-FFN call: the n-tile width of the
// single-CTA gate_up launch (256 or 128), the K splits of the gate_up
// projection (the dense layer with few tokens: split s writes its raw fp32
// accumulators at gate_up_part + s * T * 2I, and launch_swiglu_partials
// adds them and forms h), and the K splits of the down projection (split s
// writes partial rows at y_shared + s * T * H; the caller sums them).  The
// MoE layer uses the defaults.
struct FfnTiling {
  int part = 0;                    // 0: gate_up and down; 1: gate_up only; 2: down only
  int gate_up_bn = 256;
  int gate_up_ksplit = 1;
  float* gate_up_part = nullptr;   // [gate_up_ksplit][T][2I] when gate_up_ksplit > 1
  int down_ksplit = 1;
};
// swiglu.cu: h[t][j] = w * silu(g) * u from the K-split partials of gate_up
cudaError_t launch_swiglu_partials(const float* part, int ksplit, int64_t T, int I, float w,
                                   bool f16, void* h, int32_t* status, int num_sms,
                                   cudaStream_t stream);
cudaError_t launch_expert_ffn_bf16(const Layer& L, const void* x, const void* x_perm,
                                   const int32_t* offsets, const int32_t* perm_slot,
                                   const float* topk_w, const float* gamma, const void* w_gate_up,
                                   const void* w_down, const void* ws_gate_up,
                                   const void* ws_down, void* h, void* y_routed, void* y_shared,
                                   int32_t* status, int num_sms, cudaStream_t stream,
                                   bool* map_error, const FfnTiling& tiling = FfnTiling());
cudaError_t launch_router_logits_sm100(const Layer& L, const void* x, const void* w_parts,
                                       float* logits, int ld_z, int ksplit, int32_t* status,
                                       int num_sms, cudaStream_t stream, bool* map_error);

// grouped_gemm_simt.cu (fp32, CUDA cores)
cudaError_t launch_expert_ffn_f32(const Layer& L, const void* x, const void* x_perm,
                                  const int32_t* offsets, const int32_t* perm_slot,
                                  const float* topk_w, const float* gamma, const void* w_gate_up,
                                  const void* w_down, const void* ws_gate_up, const void* ws_down,
                                  void* h, void* y_routed, void* y_shared, int32_t* status,
                                  int num_sms, cudaStream_t stream);

// rmsnorm.cu (out may alias x)
cudaError_t launch_rmsnorm(int64_t T, int H, int dtype, float eps, const void* x,
                           const void* weight, void* out, int num_sms, cudaStream_t stream);

// combine.cu
cudaError_t launch_combine(const Layer& L, const void* y_routed, const void* y_shared,
                           const int32_t* inv_perm, void* out, int32_t* status, int num_sms,
                           cudaStream_t stream);

}  // namespace moe
