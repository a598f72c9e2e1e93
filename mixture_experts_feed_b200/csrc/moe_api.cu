// The C ABI of libinklingmoe.so (declared in include/inkling_moe.h): argument
// checks, workspace layout and the order of launches.  Every step of the
// layer runs in this library's kernels; there is no host compute path.
#include <atomic>
#include <mutex>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "inkling_moe.h"
#include "internal.h"

namespace moe {
namespace {

constexpr int kVersion = 1;
constexpr size_t kRegionAlign = 1024;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
  size_t status, logits, wparts, counts, chunk, topk_w, topk_idx, gamma, offsets, perm_slot, inv_perm,
      x_perm, h, y_routed, y_shared, x_norm, total;
};

// Row stride of the router logits: E+S rounded up to 32 (whole 32-column
// chunks of the tensor-core epilogue stay inside a row).
int logits_ld(const Layer& L) { return (L.E + L.S + 31) / 32 * 32; }

// K splits of the tensor-core router: enough CTAs for a B200's 148 SMs when
// T is small, at most 32.  A function of the layer shape only, so the
// partial-sum order (and every result) is the same on any device.
int router_ksplit(const Layer& L) {
  if (L.dtype != MOE_BF16) return 1;
  const int64_t tiles = (L.T + 127) / 128 * ((L.E + L.S + 159) / 160);   // router tiles
  int64_t ks = 148 / (tiles > 0 ? tiles : 1);
  if (ks < 1) ks = 1;
  if (ks > 32) ks = 32;
  return static_cast<int>(ks);
}

WsLayout ws_layout(const Layer& L) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes > 0 ? bytes : 1, kRegionAlign);
    return o;
  };
  const size_t elt = L.dtype == MOE_BF16 ? 2 : 4;
  const size_t T = static_cast<size_t>(L.T);
  const size_t Rk = T * L.k;
  const size_t Rh = Rk + T * L.S;
  w.status = take(kStatusBytes);
  w.logits = take(T * logits_ld(L) * 4 * router_ksplit(L));
  w.wparts = take(L.dtype == MOE_BF16 ? 3 * static_cast<size_t>(L.E + L.S) * L.H * 2 : 0);
  w.counts = take(static_cast<size_t>(L.E) * 4);
  w.chunk = take(static_cast<size_t>(L.E) * permute_chunks(Rk) * 4);   // per-chunk expert counts
  w.topk_w = take(Rk * 4);
  w.topk_idx = take(Rk * 4);
  w.gamma = take(T * L.S * 4);
  w.offsets = take((static_cast<size_t>(L.E) + 1) * 4);
  w.perm_slot = take(Rk * 4);
  w.inv_perm = take(Rk * 4);
  w.x_perm = take(Rk * L.H * elt);
  w.h = take(Rh * L.I * elt);
  const size_t yel = L.y_f16 ? 2 : 4;   // expert output rows: fp32, or fp16
  w.y_routed = take(Rk * L.H * yel);
  w.y_shared = take(T * L.S * L.H * yel);
  w.x_norm = take(T * L.H * elt);    // moe_forward_prenorm: the normalised input
  w.total = off;
  return w;
}

moe_status_t check_desc(const moe_layer_desc_t* d, Layer* L) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->num_tokens < 0 || d->hidden <= 0 || d->n_routed <= 0 || d->top_k <= 0 ||
      d->n_shared < 0 || d->intermediate <= 0)
    return MOE_ERR_INVALID_ARG;
  if (d->top_k > d->n_routed) return MOE_ERR_INVALID_ARG;
  if (d->dtype != MOE_F32 && d->dtype != MOE_BF16 && d->dtype != MOE_BF16_F16DOWN)
    return MOE_ERR_INVALID_ARG;
  if (!isfinite(d->route_scale) || !isfinite(d->global_scale)) return MOE_ERR_INVALID_ARG;
  if (d->top_k > 16 || d->n_routed > 1024 || d->n_shared > 8) return MOE_ERR_UNSUPPORTED;
  if (d->hidden % 64 != 0 || d->intermediate % 64 != 0) return MOE_ERR_UNSUPPORTED;
  const int64_t rows = d->num_tokens * (static_cast<int64_t>(d->top_k) + d->n_shared);
  if (d->num_tokens > (int64_t{1} << 31) / 32 || rows >= (int64_t{1} << 31))
    return MOE_ERR_UNSUPPORTED;
  L->T = d->num_tokens;
  L->H = d->hidden;
  L->E = d->n_routed;
  L->k = d->top_k;
  L->S = d->n_shared;
  L->I = d->intermediate;
  L->dtype = d->dtype == MOE_F32 ? MOE_F32 : MOE_BF16;
  L->down_f16 = d->dtype == MOE_BF16_F16DOWN;
  L->y_f16 = L->down_f16;
  L->route_scale = d->route_scale;
  L->global_scale = d->global_scale;
  return MOE_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

moe_status_t check_ws(const Layer& L, const void* ws, size_t bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOE_ERR_INVALID_ARG;
  if (bytes < ws_layout(L).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace

moe_status_t validate_desc(const moe_layer_desc_t* d, Layer* L) { return check_desc(d, L); }

int device_sm_count() {
  static std::atomic<int> cached[64];   // 0 = not queried yet; same value from any thread
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool cacheable = dev >= 0 && dev < 64;
  int n = cacheable ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    if (cacheable) cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

int num_sms() { return device_sm_count(); }

template <typename P>
P* region(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                        \
  do {                                       \
    const moe_status_t _s = (expr);          \
    if (_s != MOE_OK) return _s;             \
  } while (0)

moe_status_t route_impl(const Layer& L, const void* x, const float* w_router,
                        const float* corr_bias, float* topk_w, int32_t* topk_idx,
                        float* shared_gamma, void* ws, cudaStream_t stream) {
  const WsLayout w = ws_layout(L);
  float* logits = region<float>(ws, w.logits);
  const int ld = logits_ld(L);
  const int ksplit = router_ksplit(L);
  if (L.dtype == MOE_BF16) {
    void* parts = region<void>(ws, w.wparts);
    MOE_TRY(cuda_status(launch_router_split(L, w_router, parts, num_sms(), stream)));
    bool map_error = false;
    const cudaError_t e = launch_router_logits_sm100(L, x, parts, logits, ld, ksplit,
                                                     region<int32_t>(ws, w.status), num_sms(),
                                                     stream, &map_error);
    if (map_error) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cuda_status(e));
  } else {
    MOE_TRY(cuda_status(launch_router_logits(L, x, w_router, logits, ld, stream)));
  }
  return cuda_status(launch_router_topk(L, logits, ld, ksplit, corr_bias, topk_w, topk_idx,
                                        shared_gamma, stream));
}

moe_status_t permute_impl(const Layer& L, const int32_t* topk_idx, const uint8_t* pad,
                          const void* x, int32_t* offsets, int32_t* perm_slot, int32_t* inv_perm,
                          void* x_perm, void* ws, cudaStream_t stream) {
  const WsLayout w = ws_layout(L);
  return cuda_status(launch_permute(L, topk_idx, pad, x, offsets, perm_slot, inv_perm, x_perm,
                                    region<int32_t>(ws, w.counts), region<int32_t>(ws, w.chunk),
                                    region<int32_t>(ws, w.status),
                                    num_sms(), stream));
}

// The expert GEMMs of `L` with the activated rows in `h` (routed rows first,
// then S x T shared rows) and the status word at `status`.
moe_status_t ffn_launch(const Layer& L, const void* x, const void* x_perm, const int32_t* offsets,
                        const int32_t* perm_slot, const float* topk_w, const float* gamma,
                        const void* wgu, const void* wd, const void* wsgu, const void* wsd,
                        void* y_routed, void* y_shared, void* h, int32_t* status,
                        cudaStream_t stream) {
  if (L.dtype == MOE_BF16) {
    bool map_error = false;
    const cudaError_t e = launch_expert_ffn_bf16(L, x, x_perm, offsets, perm_slot, topk_w, gamma,
                                                 wgu, wd, wsgu, wsd, h, y_routed, y_shared,
                                                 status, num_sms(), stream, &map_error);
    if (map_error) return MOE_ERR_INVALID_ARG;
    return cuda_status(e);
  }
  return cuda_status(launch_expert_ffn_f32(L, x, x_perm, offsets, perm_slot, topk_w, gamma, wgu,
                                           wd, wsgu, wsd, h, y_routed, y_shared, status,
                                           num_sms(), stream));
}

moe_status_t ffn_impl(const Layer& L, const void* x, const void* x_perm, const int32_t* offsets,
                      const int32_t* perm_slot, const float* topk_w, const float* gamma,
                      const void* wgu, const void* wd, const void* wsgu, const void* wsd,
                      void* y_routed, void* y_shared, void* ws, cudaStream_t stream) {
  const WsLayout w = ws_layout(L);
  return ffn_launch(L, x, x_perm, offsets, perm_slot, topk_w, gamma, wgu, wd, wsgu, wsd, y_routed,
                    y_shared, region<void>(ws, w.h), region<int32_t>(ws, w.status), stream);
}

// The side stream of moe_forward on each device, with its fork and join
// events: created on first use (no device memory), kept for the life of the
// process.  A mutex orders the fork/join sequences of calls from several host
// threads, so that each record/wait pair of one call is not interleaved
// with another call's.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
SideStream g_side[kMaxSideDevices];
std::mutex g_side_mutex;

// Returns the side stream of the current device (nullptr if it cannot be made).
SideStream* side_stream() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return nullptr;
  SideStream& ss = g_side[dev];
  if (ss.stream == nullptr) {
    cudaStream_t st = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    ss.fork = f;
    ss.join = j;
    ss.stream = st;
  }
  return &ss;
}

// moe_forward with an optional RMSNorm prologue (norm_weight != null): the
// normalised input goes to the workspace and feeds every later step.
//
// bf16 layers with shared experts overlap them with the permutation: after
// the router, a fork to the side stream runs the shared experts' GEMMs (they
// need the gammas, not the permutation) while the caller's stream runs the
// permutation and the routed experts' GEMMs; the join comes before the
// combine.  The shared experts write their own activated rows (after the
// routed rows in h) and y_shared, so the two streams share no buffer.
moe_status_t forward_checked(const moe_layer_desc_t* desc, const void* x, const void* norm_weight,
                             float norm_eps, const float* w_router, const float* corr_bias,
                             const void* w_gate_up, const void* w_down, const void* ws_gate_up,
                             const void* ws_down, const uint8_t* padding_mask, void* out,
                             float* topk_w, int32_t* topk_idx, float* shared_gamma,
                             void* workspace, size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  if (!aligned16(x) || !aligned16(w_router) || corr_bias == nullptr || !aligned16(w_gate_up) ||
      !aligned16(w_down) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (L.S > 0 && (!aligned16(ws_gate_up) || !aligned16(ws_down))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  if (L.T == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(L);
  if (norm_weight != nullptr) {
    void* xn = region<void>(workspace, w.x_norm);
    MOE_TRY(cuda_status(launch_rmsnorm(L.T, L.H, L.dtype, norm_eps, x, norm_weight, xn, num_sms(), s)));
    x = xn;
  }
  float* tw = topk_w ? topk_w : region<float>(workspace, w.topk_w);
  int32_t* ti = topk_idx ? topk_idx : region<int32_t>(workspace, w.topk_idx);
  float* sg = shared_gamma ? shared_gamma : region<float>(workspace, w.gamma);
  int32_t* offsets = region<int32_t>(workspace, w.offsets);
  int32_t* perm_slot = region<int32_t>(workspace, w.perm_slot);
  int32_t* inv_perm = region<int32_t>(workspace, w.inv_perm);
  void* x_perm = region<void>(workspace, w.x_perm);
  void* y_routed = region<void>(workspace, w.y_routed);
  void* y_shared = region<void>(workspace, w.y_shared);
  MOE_TRY(route_impl(L, x, w_router, corr_bias, tw, ti, sg, workspace, s));
  SideStream* side = (L.dtype == MOE_BF16 && L.S > 0) ? side_stream() : nullptr;
  int32_t* status = region<int32_t>(workspace, w.status);
  void* h = region<void>(workspace, w.h);
  if (side != nullptr) {
    std::lock_guard<std::mutex> lock(g_side_mutex);
    MOE_TRY(cuda_status(cudaEventRecord(side->fork, s)));
    MOE_TRY(cuda_status(cudaStreamWaitEvent(side->stream, side->fork, 0)));
    // the shared groups' gate_up alone (E = 0, k = 0), their h rows after
    // the routed ones
    Layer Ls = L;
    Ls.E = 0;
    Ls.k = 0;
    void* h_shared = static_cast<uint8_t*>(h) + static_cast<size_t>(L.T) * L.k * L.I * 2;
    FfnTiling gate_up_only;
    gate_up_only.part = 1;
    bool map_error = false;
    const cudaError_t e = launch_expert_ffn_bf16(Ls, x, x, nullptr, nullptr, nullptr, sg, nullptr,
                                                 nullptr, ws_gate_up, ws_down, h_shared, y_shared,
                                                 y_shared, status, num_sms(), side->stream,
                                                 &map_error, gate_up_only);
    if (map_error) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cuda_status(e));
    MOE_TRY(cuda_status(cudaEventRecord(side->join, side->stream)));
  }
  // the permuted copy of x: the GEMM's A tiles are then whole TMA boxes (the
  // row-gathering mode, x_perm = null, issues one TMA per 4 rows and runs
  // slower once tiles are full)
  MOE_TRY(permute_impl(L, ti, padding_mask, x, offsets, perm_slot, inv_perm, x_perm, workspace, s));
  if (side == nullptr) {
    MOE_TRY(ffn_launch(L, x, x_perm, offsets, perm_slot, tw, sg, w_gate_up, w_down, ws_gate_up,
                       ws_down, y_routed, y_shared, h, status, s));
  } else {
    // the routed groups' gate_up; then, once the shared gate_up has joined,
    // one down projection over all groups (routed and shared rows of h)
    Layer Lr = L;
    Lr.S = 0;
    FfnTiling gate_up_only, down_only;
    gate_up_only.part = 1;
    down_only.part = 2;
    bool map_error = false;
    cudaError_t e = launch_expert_ffn_bf16(Lr, x, x_perm, offsets, perm_slot, tw, sg, w_gate_up,
                                           w_down, ws_gate_up, ws_down, h, y_routed, y_shared,
                                           status, num_sms(), s, &map_error, gate_up_only);
    if (map_error) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cuda_status(e));
    {
      std::lock_guard<std::mutex> lock(g_side_mutex);
      MOE_TRY(cuda_status(cudaStreamWaitEvent(s, side->join, 0)));
    }
    e = launch_expert_ffn_bf16(L, x, x_perm, offsets, perm_slot, tw, sg, w_gate_up, w_down,
                               ws_gate_up, ws_down, h, y_routed, y_shared, status, num_sms(), s,
                               &map_error, down_only);
    if (map_error) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cuda_status(e));
  }
  return cuda_status(launch_combine(L, y_routed, y_shared, inv_perm, out, status, num_sms(), s));
}

// ------------------------------------------------------------ dense layer
// InklingDenseMLP runs through the expert GEMMs as one shared group over all
// T tokens (E = 0, S = 1) whose per-token weight is global_scale, then the
// recombination with k = 0 rounds y into out.
struct DenseWs {
  size_t status, h, y, gu_part, x_norm, total;
};

// Tile choices of the dense layer on the tensor cores (functions of the
// shape only, so every device computes the same partial sums).  With few
// token rows (decode) the layer streams its weights: the single-CTA gate_up
// launch takes 128-wide n-tiles when that fills the 148 SMs better, and the
// down projection splits K until its tiles reach about 148.
constexpr int kTilingSms = 148;

FfnTiling dense_tiling(const Layer& L) {
  FfnTiling t;
  if (L.dtype != MOE_BF16 || L.T <= 0) return t;
  const int64_t mt = (L.T + 127) / 128;
  auto waves_eff = [](int64_t tiles) {
    const int64_t waves = (tiles + kTilingSms - 1) / kTilingSms;
    return static_cast<double>(tiles) / static_cast<double>(waves * kTilingSms);
  };
  if (L.T <= 128) {   // every tile on the single-CTA launch
    const int64_t t256 = mt * ((2 * L.I + 255) / 256), t128 = mt * ((2 * L.I + 127) / 128);
    double best = waves_eff(t256);
    if (t256 < 4 * kTilingSms && waves_eff(t128) > best + 0.05) {
      t.gate_up_bn = 128;
      best = waves_eff(t128);
    }
    // or split gate_up's K (256-wide tiles, each split a fresh accumulation,
    // at least 16 K blocks a split) when that fills the waves better still
    for (int ks = 2; ks <= 4 && t256 < 4 * kTilingSms; ++ks) {
      if (L.H / 64 / ks < 16) break;
      if (waves_eff(t256 * ks) > best + 0.05) {
        best = waves_eff(t256 * ks);
        t.gate_up_ksplit = ks;
        t.gate_up_bn = 256;
      }
    }
  }
  const int64_t down_tiles = mt * ((L.H + 255) / 256);   // m-tiles x n-tiles (either launch)
  if (down_tiles < kTilingSms) {
    int64_t ks = kTilingSms / down_tiles;
    const int64_t kmax = L.I / 64 / 4;                     // at least 4 K blocks per split
    if (ks > kmax) ks = kmax;
    if (ks > 16) ks = 16;
    t.down_ksplit = static_cast<int>(ks < 1 ? 1 : ks);
  }
  return t;
}

moe_status_t check_dense(const moe_dense_desc_t* d, Layer* L) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->num_tokens < 0 || d->hidden <= 0 || d->intermediate <= 0) return MOE_ERR_INVALID_ARG;
  if (d->dtype != MOE_F32 && d->dtype != MOE_BF16 && d->dtype != MOE_BF16_F16DOWN)
    return MOE_ERR_INVALID_ARG;
  if (!isfinite(d->global_scale)) return MOE_ERR_INVALID_ARG;
  if (d->hidden % 64 != 0 || d->intermediate % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (d->num_tokens >= (int64_t{1} << 26)) return MOE_ERR_UNSUPPORTED;
  L->T = d->num_tokens;
  L->H = d->hidden;
  L->E = 0;
  L->k = 0;
  L->S = 1;
  L->I = d->intermediate;
  L->dtype = d->dtype == MOE_F32 ? MOE_F32 : MOE_BF16;
  L->down_f16 = d->dtype == MOE_BF16_F16DOWN;
  L->route_scale = 1.0f;
  L->global_scale = d->global_scale;
  return MOE_OK;
}

DenseWs dense_ws_layout(const Layer& L) {
  DenseWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes > 0 ? bytes : 1, kRegionAlign);
    return o;
  };
  const size_t elt = L.dtype == MOE_BF16 ? 2 : 4;
  const size_t T = static_cast<size_t>(L.T);
  w.status = take(kStatusBytes);
  w.h = take(T * L.I * elt);
  const FfnTiling tiling = dense_tiling(L);
  w.y = take(T * L.H * 4 * tiling.down_ksplit);   // one partial per K split
  // gate_up's K-split accumulators (fp32, [ks][T][2I]) when its K is split
  w.gu_part = take(tiling.gate_up_ksplit > 1 ? T * 2 * L.I * 4 * tiling.gate_up_ksplit : 0);
  w.x_norm = take(T * L.H * elt);    // moe_dense_mlp_prenorm: the normalised input
  w.total = off;
  return w;
}

moe_status_t dense_checked(const moe_dense_desc_t* desc, const void* x, const void* norm_weight,
                           float norm_eps, const void* w_gate_up, const void* w_down, void* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_dense(desc, &L));
  if (L.T == 0) return MOE_OK;   // nothing to read or write
  if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return MOE_ERR_INVALID_ARG;
  const DenseWs w = dense_ws_layout(L);
  if (workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = region<int32_t>(workspace, w.status);
  void* h = region<void>(workspace, w.h);
  float* y = region<float>(workspace, w.y);
  if (norm_weight != nullptr) {
    void* xn = region<void>(workspace, w.x_norm);
    MOE_TRY(cuda_status(launch_rmsnorm(L.T, L.H, L.dtype, norm_eps, x, norm_weight, xn, num_sms(), s)));
    x = xn;
  }
  // one shared group: the routed operands are never read (E = 0, k = 0)
  FfnTiling tiling = dense_tiling(L);
  tiling.gate_up_part = region<float>(workspace, w.gu_part);
  if (L.dtype == MOE_BF16) {
    bool map_error = false;
    const cudaError_t e = launch_expert_ffn_bf16(L, x, x, nullptr, nullptr, nullptr, nullptr,
                                                 nullptr, nullptr, w_gate_up, w_down, h, y, y,
                                                 status, num_sms(), s, &map_error, tiling);
    if (map_error) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cuda_status(e));
  } else {
    MOE_TRY(cuda_status(launch_expert_ffn_f32(L, x, x, nullptr, nullptr, nullptr, nullptr,
                                              nullptr, nullptr, w_gate_up, w_down, h, y, y,
                                              status, num_sms(), s)));
  }
  // the recombination sums the K-split partials in split order (S of them)
  Layer Lc = L;
  Lc.S = tiling.down_ksplit;
  return cuda_status(launch_combine(Lc, y, y, nullptr, out, status, num_sms(), s));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_workspace_size(const moe_layer_desc_t* desc, size_t* bytes) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *bytes = ws_layout(L).total;
  return MOE_OK;
}

moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || workspace_bytes < kStatusBytes) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_read_device_status(void* workspace, void* stream, int32_t* device_code) {
  if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t code = 0;
  MOE_TRY(cuda_status(cudaMemcpyAsync(&code, workspace, sizeof(code), cudaMemcpyDeviceToHost, s)));
  MOE_TRY(cuda_status(cudaStreamSynchronize(s)));
  MOE_TRY(cuda_status(cudaMemsetAsync(workspace, 0, sizeof(code), s)));
  if (device_code != nullptr) *device_code = code;
  if (code == 0) return MOE_OK;
  return code == DEV_WAIT_TIMEOUT ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE_CHECK;
}

moe_status_t moe_route(const moe_layer_desc_t* desc, const void* x, const float* w_router,
                       const float* corr_bias, float* topk_w, int32_t* topk_idx,
                       float* shared_gamma, void* workspace, size_t workspace_bytes,
                       void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  if (!aligned16(x) || !aligned16(w_router) || corr_bias == nullptr || topk_w == nullptr ||
      topk_idx == nullptr || (L.S > 0 && shared_gamma == nullptr))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  if (L.T == 0) return MOE_OK;
  return route_impl(L, x, w_router, corr_bias, topk_w, topk_idx, shared_gamma, workspace,
                    static_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(const moe_layer_desc_t* desc, const int32_t* topk_idx,
                         const uint8_t* padding_mask, const void* x, int32_t* expert_offsets,
                         int32_t* perm_slot, int32_t* inv_perm, void* x_perm, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  // x_perm null: no row gather (x is then not read and may be null)
  if (topk_idx == nullptr || expert_offsets == nullptr || perm_slot == nullptr ||
      inv_perm == nullptr || (x_perm != nullptr && (!aligned16(x) || !aligned16(x_perm))))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L.T == 0) {
    return cuda_status(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (L.E + 1), s));
  }
  return permute_impl(L, topk_idx, padding_mask, x, expert_offsets, perm_slot, inv_perm, x_perm,
                      workspace, s);
}

moe_status_t moe_expert_ffn(const moe_layer_desc_t* desc, const void* x, const void* x_perm,
                            const int32_t* expert_offsets, const int32_t* perm_slot,
                            const float* topk_w, const float* shared_gamma,
                            const void* w_gate_up, const void* w_down, const void* ws_gate_up,
                            const void* ws_down, void* y_routed, void* y_shared,
                            void* workspace, size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  // perm_slot may be NULL only with x_perm given: rows already in slot order
  if (!aligned16(x) || (x_perm != nullptr && !aligned16(x_perm)) || expert_offsets == nullptr ||
      (perm_slot == nullptr && x_perm == nullptr) || topk_w == nullptr || !aligned16(w_gate_up) ||
      !aligned16(w_down) || !aligned16(y_routed))
    return MOE_ERR_INVALID_ARG;
  if (L.S > 0 && (shared_gamma == nullptr || !aligned16(ws_gate_up) || !aligned16(ws_down) ||
                  !aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  if (L.T == 0) return MOE_OK;
  return ffn_impl(L, x, x_perm, expert_offsets, perm_slot, topk_w, shared_gamma, w_gate_up, w_down,
                  ws_gate_up, ws_down, y_routed, y_shared, workspace,
                  static_cast<cudaStream_t>(stream));
}

moe_status_t moe_shared_ffn(const moe_layer_desc_t* desc, const void* x, const float* shared_gamma,
                            const void* ws_gate_up, const void* ws_down, void* y_shared,
                            void* workspace, size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  if (L.S == 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || shared_gamma == nullptr || !aligned16(ws_gate_up) || !aligned16(ws_down) ||
      !aligned16(y_shared))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  if (L.T == 0) return MOE_OK;
  // the S shared groups alone: no routed group (E = 0, k = 0)
  const WsLayout w = ws_layout(L);
  Layer Ls = L;
  Ls.E = 0;
  Ls.k = 0;
  void* h = region<void>(workspace, w.h);
  int32_t* status = region<int32_t>(workspace, w.status);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L.dtype == MOE_BF16) {
    bool map_error = false;
    const cudaError_t e = launch_expert_ffn_bf16(Ls, x, x, nullptr, nullptr, nullptr, shared_gamma,
                                                 nullptr, nullptr, ws_gate_up, ws_down, h, y_shared,
                                                 y_shared, status, num_sms(), s, &map_error);
    if (map_error) return MOE_ERR_INVALID_ARG;
    return cuda_status(e);
  }
  return cuda_status(launch_expert_ffn_f32(Ls, x, x, nullptr, nullptr, nullptr, shared_gamma,
                                           nullptr, nullptr, ws_gate_up, ws_down, h, y_shared,
                                           y_shared, status, num_sms(), s));
}

int32_t moe_shared_ffn_kernel_count(const moe_layer_desc_t* desc) {
  Layer L;
  if (check_desc(desc, &L) != MOE_OK || L.T == 0 || L.S == 0) return 0;
  return 2;   // gate_up + down, each one launch (all S groups have T rows)
}

moe_status_t moe_combine(const moe_layer_desc_t* desc, const void* y_routed, const void* y_shared,
                         const int32_t* inv_perm, void* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Layer L;
  MOE_TRY(check_desc(desc, &L));
  if (!aligned16(y_routed) || inv_perm == nullptr || !aligned16(out) ||
      (L.S > 0 && !aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(L, workspace, workspace_bytes));
  if (L.T == 0) return MOE_OK;
  const WsLayout w = ws_layout(L);
  return cuda_status(launch_combine(L, y_routed, y_shared, inv_perm, out,
                                    region<int32_t>(workspace, w.status), num_sms(),
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward(const moe_layer_desc_t* desc, const void* x, const float* w_router,
                         const float* corr_bias, const void* w_gate_up, const void* w_down,
                         const void* ws_gate_up, const void* ws_down, const uint8_t* padding_mask,
                         void* out, float* topk_w, int32_t* topk_idx, float* shared_gamma,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return forward_checked(desc, x, nullptr, 0.0f, w_router, corr_bias, w_gate_up, w_down,
                         ws_gate_up, ws_down, padding_mask, out, topk_w, topk_idx, shared_gamma,
                         workspace, workspace_bytes, stream);
}

moe_status_t moe_forward_prenorm(const moe_layer_desc_t* desc, const void* x,
                                 const void* norm_weight, float norm_eps, const float* w_router,
                                 const float* corr_bias, const void* w_gate_up, const void* w_down,
                                 const void* ws_gate_up, const void* ws_down,
                                 const uint8_t* padding_mask, void* out, float* topk_w,
                                 int32_t* topk_idx, float* shared_gamma, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!aligned16(norm_weight) || !isfinite(norm_eps) || norm_eps < 0.0f) return MOE_ERR_INVALID_ARG;
  return forward_checked(desc, x, norm_weight, norm_eps, w_router, corr_bias, w_gate_up, w_down,
                         ws_gate_up, ws_down, padding_mask, out, topk_w, topk_idx, shared_gamma,
                         workspace, workspace_bytes, stream);
}

moe_status_t moe_rmsnorm(int64_t num_tokens, int32_t hidden, moe_dtype_t dtype, float eps,
                         const void* x, const void* weight, void* out, void* stream) {
  if (num_tokens < 0 || hidden <= 0 || (dtype != MOE_F32 && dtype != MOE_BF16) ||
      !isfinite(eps) || eps < 0.0f)
    return MOE_ERR_INVALID_ARG;
  if (hidden % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (num_tokens == 0) return MOE_OK;
  if (!aligned16(x) || !aligned16(weight) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_rmsnorm(num_tokens, hidden, dtype, eps, x, weight, out, num_sms(),
                                    static_cast<cudaStream_t>(stream)));
}

int32_t moe_forward_kernel_count(const moe_layer_desc_t* desc) {
  Layer L;
  if (check_desc(desc, &L) != MOE_OK || L.T == 0) return 0;
  // router: (bf16: split + tensor-core logits | fp32: logits) + top-k (plus
  // a partial-logit sum when K is split 4 or more ways); permute: chunk
  // counts, chunk scan, scatter (one kernel for at most 256 slots), row
  // gather; experts: gate_up + down (bf16
  // with T > 128: CTA-pair launch + single-CTA launch each; bf16 with shared
  // experts: their gate_up on the side stream too, their down in the routed
  // experts' down launches); combine.
  const int experts = L.dtype == MOE_BF16 ? (L.T > 128 ? 4 : 2) + (L.S > 0 ? 1 : 0) : 2;
  return (L.dtype == MOE_BF16 ? 2 : 1) + router_topk_launches(router_ksplit(L), L.T) +
         permute_kernel_count(L.T * L.k, true) + experts + 1;
}

moe_status_t moe_dense_workspace_size(const moe_dense_desc_t* desc, size_t* bytes) {
  Layer L;
  MOE_TRY(check_dense(desc, &L));
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *bytes = dense_ws_layout(L).total;
  return MOE_OK;
}

moe_status_t moe_dense_mlp(const moe_dense_desc_t* desc, const void* x, const void* w_gate_up,
                           const void* w_down, void* out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return dense_checked(desc, x, nullptr, 0.0f, w_gate_up, w_down, out, workspace, workspace_bytes,
                       stream);
}

moe_status_t moe_dense_mlp_prenorm(const moe_dense_desc_t* desc, const void* x,
                                   const void* norm_weight, float norm_eps, const void* w_gate_up,
                                   const void* w_down, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!aligned16(norm_weight) || !isfinite(norm_eps) || norm_eps < 0.0f) return MOE_ERR_INVALID_ARG;
  return dense_checked(desc, x, norm_weight, norm_eps, w_gate_up, w_down, out, workspace,
                       workspace_bytes, stream);
}

int32_t moe_dense_kernel_count(const moe_dense_desc_t* desc) {
  Layer L;
  if (check_dense(desc, &L) != MOE_OK || L.T == 0) return 0;
  // gate_up + down (one launch each: the one group's tiles are all CTA-pair
  // or all single-CTA tiles; a K-split gate_up adds its SwiGLU pass), then
  // the rounding pass
  return L.dtype == MOE_BF16 && dense_tiling(L).gate_up_ksplit > 1 ? 4 : 3;
}

int32_t moe_dense_prenorm_kernel_count(const moe_dense_desc_t* desc) {
  const int32_t n = moe_dense_kernel_count(desc);
  return n > 0 ? n + 1 : 0;   // + the RMSNorm prologue
}

int32_t moe_forward_prenorm_kernel_count(const moe_layer_desc_t* desc) {
  const int32_t n = moe_forward_kernel_count(desc);
  return n > 0 ? n + 1 : 0;   // + the RMSNorm prologue
}

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported layer shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side index check failed";
    case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

int32_t moe_version(void) { return kVersion; }

}  // extern "C"
