// Grouped expert GEMMs in fp32 on the CUDA cores, for layers whose dtype is
// fp32.  Same groups, tile order and fused epilogues as the tensor-core path
// (grouped_gemm_sm100.cu), but exact fp32 FFMA: tf32 tensor-core inputs would
// round every operand to 10 mantissa bits, which an fp32 layer cannot accept.
// Tiles of 64 rows x 64 columns x 16 K; 256 threads, 4 x 4 outputs each.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "grouping.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int SB_M = 64, SB_N = 64, SB_K = 16, SB_THREADS = 256;

struct SimtParams {
  const float* A[2];
  const float* B[2];
  float* out[2];
  const int32_t* offsets;
  const int32_t* perm_slot;
  const float* topk_w;
  const float* gamma;   // null: every shared row gets uniform_w (the dense layer)
  float uniform_w;
  int32_t* status;
  int64_t T, a1_base, a1_stride;
  int E, S, K, N, ld_out, rows_cap;
  int gather_k;   // gate_up: > 0 = routed row r reads x[perm_slot[r] / gather_k] (A[0] = x)
};

template <bool GATE_UP>
__global__ void __launch_bounds__(SB_THREADS) grouped_gemm_simt_kernel(const SimtParams p) {
  __shared__ __align__(16) float As[SB_K][SB_M + 4];
  __shared__ __align__(16) float Bs[SB_K][SB_N + 4];
  __shared__ int s_bad;
  extern __shared__ int s_tables[];
  int* s_off = s_tables;
  int* s_tile = s_tables + p.E + 1;
  const int G = p.E + p.S;
  const int n_tiles = (p.N + SB_N - 1) / SB_N;
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  if (tid < 32) build_tile_prefix(p.offsets, p.E, p.S, p.T, kAllTiles, SB_M, n_tiles, p.rows_cap, s_off, s_tile, &s_bad);
  __syncthreads();
  if (tid == 0 && s_bad) record_status(p.status, DEV_BAD_ROW);
  const int total = s_tile[G];
  const int tx = tid & 15, ty = tid >> 4;
  const int lr = tid >> 2, lk = (tid & 3) * 4;

  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    int g, m, n;
    decode_tile(tile, s_tile, G, s_off, p.E, p.T, kAllTiles, SB_M, g, m, n);
    const GroupInfo gi = group_info(g, s_off, p.E, p.T, p.a1_base, p.a1_stride);
    const float* A = p.A[gi.src];
    const float* B = p.B[gi.src] + static_cast<int64_t>(gi.b_idx) * p.N * p.K;
    const bool a_ok = m * SB_M + lr < gi.rows;
    const bool b_ok = n * SB_N + lr < p.N;
    int64_t a_src = gi.a_row0 + m * SB_M + (a_ok ? lr : 0);
    if (GATE_UP && p.gather_k > 0 && gi.src == 0) {
      // gathered routed rows: the row's token; rows past the group read token 0
      int tok = 0;
      if (a_ok) {
        const int slot = p.perm_slot[a_src];
        if (slot >= 0 && slot < p.rows_cap) tok = slot / p.gather_k;
        else record_status(p.status, DEV_BAD_ROW);
      }
      a_src = tok;
    }
    const float* ap = A + a_src * p.K + lk;
    const float* bp = B + static_cast<int64_t>(n * SB_N + (b_ok ? lr : 0)) * p.K + lk;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    for (int k0 = 0; k0 < p.K; k0 += SB_K) {
      const float4 av = a_ok ? *reinterpret_cast<const float4*>(ap + k0) : make_float4(0, 0, 0, 0);
      const float4 bv = b_ok ? *reinterpret_cast<const float4*>(bp + k0) : make_float4(0, 0, 0, 0);
      __syncthreads();
      As[lk + 0][lr] = av.x; As[lk + 1][lr] = av.y; As[lk + 2][lr] = av.z; As[lk + 3][lr] = av.w;
      Bs[lk + 0][lr] = bv.x; Bs[lk + 1][lr] = bv.y; Bs[lk + 2][lr] = bv.z; Bs[lk + 3][lr] = bv.w;
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < SB_K; ++kk) {
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
    const int c0 = n * SB_N + tx * 4;
    if (c0 < p.N) {
      float* out = p.out[gi.src];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = m * SB_M + ty * 4 + i;
        if (r >= gi.rows) continue;
        const int64_t orow = gi.out_row0 + r;
        if (GATE_UP) {
          float w;
          if (gi.src == 0) {
            // no perm_slot: the rows are already in slot order (row r is slot r)
            const int slot = p.perm_slot != nullptr ? p.perm_slot[gi.a_row0 + r]
                                                    : static_cast<int>(gi.a_row0 + r);
            if (slot >= 0 && slot < p.rows_cap) {
              w = p.topk_w[slot];
            } else {
              record_status(p.status, DEV_BAD_ROW);
              w = 0.0f;
            }
          } else {
            w = p.gamma != nullptr ? p.gamma[static_cast<int64_t>(r) * p.S + gi.s] : p.uniform_w;
          }
          float2 hv;
          hv.x = w * (acc[i][0] / (1.0f + expf(-acc[i][0]))) * acc[i][1];
          hv.y = w * (acc[i][2] / (1.0f + expf(-acc[i][2]))) * acc[i][3];
          *reinterpret_cast<float2*>(out + orow * p.ld_out + c0 / 2) = hv;
        } else {
          *reinterpret_cast<float4*>(out + orow * p.ld_out + c0) =
              make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_expert_ffn_f32(const Layer& L, const void* x, const void* x_perm,
                                  const int32_t* offsets, const int32_t* perm_slot,
                                  const float* topk_w, const float* gamma, const void* w_gate_up,
                                  const void* w_down, const void* ws_gate_up, const void* ws_down,
                                  void* h, void* y_routed, void* y_shared, int32_t* status,
                                  int num_sms, cudaStream_t stream) {
  const int64_t Rk = L.T * L.k;
  float* hf = static_cast<float*>(h);
  const int tables = static_cast<int>(sizeof(int)) * (2 * L.E + L.S + 2);
  const unsigned grid = static_cast<unsigned>(num_sms * 4);

  SimtParams g{};
  // with x_perm null the routed rows are read from x through perm_slot
  g.A[0] = static_cast<const float*>(x_perm != nullptr ? x_perm : x);
  g.gather_k = x_perm != nullptr ? 0 : L.k;
  g.A[1] = static_cast<const float*>(x);
  g.B[0] = static_cast<const float*>(w_gate_up);
  g.B[1] = L.S > 0 ? static_cast<const float*>(ws_gate_up) : g.B[0];
  g.out[0] = hf;
  g.out[1] = hf + Rk * L.I;
  g.offsets = offsets; g.perm_slot = perm_slot; g.topk_w = topk_w; g.gamma = gamma;
  g.uniform_w = L.global_scale;
  g.status = status;
  g.T = L.T; g.a1_base = 0; g.a1_stride = 0;
  g.E = L.E; g.S = L.S; g.K = L.H; g.N = 2 * L.I; g.ld_out = L.I;
  g.rows_cap = static_cast<int>(Rk);
  const cudaError_t e =
      launch_chained(grouped_gemm_simt_kernel<true>, grid, SB_THREADS, tables, stream, g);
  if (e != cudaSuccess) return e;

  SimtParams d{};
  d.A[0] = hf;
  d.A[1] = hf;
  d.B[0] = static_cast<const float*>(w_down);
  d.B[1] = L.S > 0 ? static_cast<const float*>(ws_down) : d.B[0];
  d.out[0] = static_cast<float*>(y_routed);
  d.out[1] = static_cast<float*>(y_shared);
  d.offsets = offsets; d.perm_slot = perm_slot; d.topk_w = topk_w; d.gamma = gamma;
  d.uniform_w = L.global_scale;
  d.status = status;
  d.T = L.T; d.a1_base = Rk; d.a1_stride = L.T;
  d.E = L.E; d.S = L.S; d.K = L.I; d.N = L.H; d.ld_out = L.H;
  d.rows_cap = static_cast<int>(Rk);
  return launch_chained(grouped_gemm_simt_kernel<false>, grid, SB_THREADS, tables, stream, d);
}

}  // namespace moe
