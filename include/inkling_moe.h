/*
 * inkling_moe.h — C ABI of libinklingmoe.so, the B200 (sm_100a) forward pass
 * of the Inkling mixture-of-experts feed-forward layer.
 *
 * The layer, as the NeMo AutoModel Inkling pages state it ("layers" page):
 *   - InklingGate: fp32 router logits over a gate weight bank of E routed rows
 *     followed by S shared rows; selection of k experts by sigmoid score plus
 *     the fp32 correction bias (InklingCorrectionBias); output weights from a
 *     softmax over the log-sigmoid of the k selected routed logits
 *     concatenated with the S shared logits, times route_scale*global_scale.
 *     The first k weights go to the routed experts, the last S (the gammas)
 *     to the always-on shared experts.
 *   - InklingSharedExperts: every token through every shared expert, each
 *     output weighted by its gamma, summed.
 *   - routed experts: fused gate/up projection whose output interleaves
 *     gate and up channels ([g0, u0, g1, u1, ...]), SwiGLU scaled by the
 *     routing weight (inkling_swiglu), down projection.
 *   - InklingMoE.forward: shared plus routed, recombined per token; leading
 *     dims of the input are flattened to tokens by the caller; padded tokens
 *     never reach a routed expert.
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned DEVICE buffers, row-major and contiguous,
 *     16-byte aligned.  The library never allocates or frees memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL means the legacy default stream).  The host-side argument check
 *     runs before any launch; a non-OK return means nothing was launched
 *     (MOE_ERR_CUDA: a launch was attempted and CUDA reported an error).
 *   - Weights use the checkpoint's [out_features, in_features] orientation
 *     (the pages keep the fused projection in the checkpoint's layout, which
 *     loading reaches through a transposed view):
 *       w_router   [E+S, H] fp32    rows 0..E-1 routed, E..E+S-1 shared
 *       corr_bias  [E]      fp32
 *       w_gate_up  [E, 2I, H]       row 2j = gate_j, row 2j+1 = up_j
 *       w_down     [E, H, I]
 *       ws_gate_up [S, 2I, H], ws_down [S, H, I]   (shared experts)
 *     x, the expert weights, x_perm and out share `dtype` (MOE_BF16_F16DOWN:
 *     bf16, with w_down and ws_down fp16); the expert output rows
 *     y_routed / y_shared are fp32 (MOE_BF16_F16DOWN: fp16); moe_combine
 *     sums them in fp32 and rounds once.
 *   - Sizes: T = num_tokens, H = hidden, E = n_routed, k = top_k,
 *     S = n_shared, I = intermediate.  Limits: 1 <= k <= min(E, 16),
 *     E <= 1024, S <= 8, H % 64 == 0, I % 64 == 0, T <= 2^26,
 *     T*(k+S) < 2^31 (else MOE_ERR_UNSUPPORTED).
 *     T = 0 is accepted and launches nothing.
 *   - `workspace` is a device buffer of at least moe_workspace_size() bytes.
 *     Its first 256 bytes hold a sticky device status word; zero them once
 *     with moe_workspace_init() before first use.  Kernels that detect a bad
 *     index or a stalled pipeline record it there instead of faulting;
 *     moe_read_device_status() reads and clears it.  Bytes 64..71 of that
 *     region are the expert GEMMs' tile counters, which every call that uses
 *     them zeroes itself on its stream.
 *   - Calls sharing one workspace must be ordered on one stream.
 *   - Kernels are launched with programmatic stream serialisation: a
 *     kernel's CTAs may start while the kernel before it on the stream
 *     (this library's or the caller's) is still finishing, but they read and
 *     write global memory only after that kernel has completed and its
 *     writes are visible.  Stream order is therefore exactly that of plain
 *     launches; only the launch latency and each kernel's set-up overlap.
 */
#ifndef INKLING_MOE_H
#define INKLING_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer */
  MOE_ERR_UNSUPPORTED = 2,   /* valid layer outside this library's limits */
  MOE_ERR_WORKSPACE = 3,     /* workspace smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,          /* the CUDA runtime reported an error */
  MOE_ERR_DEVICE_CHECK = 5,  /* a kernel saw an out-of-range index */
  MOE_ERR_TIMEOUT = 6        /* a kernel's bounded pipeline wait expired */
} moe_status_t;

/*
 * Layer dtypes.
 *   MOE_F32           everything fp32; the expert GEMMs run in fp32 on the
 *                     CUDA cores.
 *   MOE_BF16          x, out and every expert weight bf16; the activated
 *                     rows h are rounded to bf16 before the down projection.
 *   MOE_BF16_F16DOWN  x, out, the router input and the gate_up weights bf16,
 *                     as MOE_BF16; the down projections' weights (w_down,
 *                     ws_down) fp16, and the activated rows h rounded to
 *                     fp16, 8 times finer than bf16; the expert output rows
 *                     y are stored in fp16 too (half the bytes of fp32).
 *                     The fp16 weights are
 *                     the checkpoint's bf16 values copied once with
 *                     moe_convert_bf16_to_f16 (exact for |w| in [2^-17, 65504]
 *                     and zero; smaller values change by at most 2^-25).
 *                     With bf16 h the rounding of h adds up to
 *                     about 1% of the output's RMS to the error of the final
 *                     bf16 rounding (1.7% of RMS when outputs reach 6 x RMS);
 *                     with fp16 h and fp16 y rows about 0.1–0.2%.  An h or y
 *                     value at or beyond 65520 in magnitude (an fp16
 *                     infinity) is recorded in the workspace status word
 *                     (MOE_ERR_DEVICE_CHECK).
 */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_BF16_F16DOWN = 2 } moe_dtype_t;

/* Layer description (the MoE fields of InklingTextConfig, with T added). */
typedef struct {
  int64_t num_tokens;    /* T: product of the input's leading dims */
  int32_t hidden;        /* H: hidden_size */
  int32_t n_routed;      /* E: n_routed_experts */
  int32_t top_k;         /* k: num_experts_per_tok */
  int32_t n_shared;      /* S: n_shared_experts */
  int32_t intermediate;  /* I: moe_intermediate_size (shared experts too) */
  int32_t dtype;         /* moe_dtype_t of x, expert weights and outputs */
  float route_scale;     /* route_scale */
  float global_scale;    /* the gate's global_scale parameter (1.0 at init) */
} moe_layer_desc_t;

/* Workspace bytes every entry point below accepts for this layer. */
moe_status_t moe_workspace_size(const moe_layer_desc_t* desc, size_t* bytes);

/* Zero the device status word at the head of `workspace` (async). */
moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Read the device status word (synchronises `stream`), then clear it.
 * Returns MOE_OK, MOE_ERR_DEVICE_CHECK or MOE_ERR_TIMEOUT; `*device_code`
 * receives the raw word (0 when clean; may be NULL). */
moe_status_t moe_read_device_status(void* workspace, void* stream, int32_t* device_code);

/*
 * moe_route — InklingGate.forward (layers page, InklingGate docstring;
 * InklingCorrectionBias.forward).
 *   x            [T, H]    dtype
 *   w_router     [E+S, H]  fp32
 *   corr_bias    [E]       fp32 (selection only)
 *   topk_w       [T, k]    fp32 out: routed weights, best expert first
 *   topk_idx     [T, k]    int32 out: expert ids by descending score
 *                          sigmoid(z)+bias; ties go to the lower id
 *   shared_gamma [T, S]    fp32 out (may be NULL when S == 0)
 * Logits are computed in fp32.  Sum over a token of topk_w and shared_gamma
 * equals route_scale*global_scale.
 */
moe_status_t moe_route(const moe_layer_desc_t* desc, const void* x, const float* w_router,
                       const float* corr_bias, float* topk_w, int32_t* topk_idx,
                       float* shared_gamma, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * moe_permute — grouped dispatch order for the routed experts (layers page,
 * InklingMoE docstring: grouped routed experts; InklingMoE.forward: padded
 * tokens never reach a routed expert).  Every live (token t, choice j)
 * pair becomes one row; rows are ordered by (expert, token) ascending.
 *   topk_idx       [T, k] int32 in, values in [0, E)
 *   padding_mask   [T] uint8 (nonzero = padded) or NULL
 *   x              [T, H] dtype in (not read, and may be NULL, when x_perm is NULL)
 *   expert_offsets [E+1] int32 out: rows of expert e are [off[e], off[e+1])
 *   perm_slot      [T*k] int32 out: for row r < off[E], the slot t*k+j it holds
 *   inv_perm       [T*k] int32 out: for slot t*k+j, its row, or -1 if padded
 *   x_perm         [T*k, H] dtype out: row r = x[perm_slot[r] / k]; or NULL:
 *                  no row copy (moe_expert_ffn can gather the rows itself)
 * The order is deterministic (no atomics decide it).
 */
moe_status_t moe_permute(const moe_layer_desc_t* desc, const int32_t* topk_idx,
                         const uint8_t* padding_mask, const void* x, int32_t* expert_offsets,
                         int32_t* perm_slot, int32_t* inv_perm, void* x_perm, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * moe_permute_noalloc — moe_permute without a workspace, for callers that
 * cannot allocate device memory (for example a plugin inside an inference
 * engine that plans all device memory ahead of time and forbids allocation
 * in its enqueue step, or a process held to a fixed device-memory budget).
 * The pages have no counterpart of this entry point; it is an addition for
 * such callers.  Arguments, outputs and results are those of moe_permute.
 *   - The per-expert counters live in a static device array of 1024 int32
 *     (4 KiB) that every GPU loading the library keeps until exit, so
 *     E must be <= 1024 (else MOE_ERR_UNSUPPORTED).
 *   - The first call on a device looks up that array's device address (a
 *     one-time set-up per device) and keeps it for the life of the process;
 *     make that first call before any stream capture, and do not call
 *     cudaDeviceReset on that device between calls (a reset would leave the
 *     kept address pointing at memory the library no longer owns).
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears it on `stream` first.  Calls that overlap on the GPU
 *     (other streams or threads) race on it: order them.
 *   - With no status word, an out-of-range expert id is skipped (its slot
 *     gets inv_perm = -1) but not reported.
 * It allocates nothing (no cudaMalloc, no cudaFree).
 */
moe_status_t moe_permute_noalloc(const moe_layer_desc_t* desc, const int32_t* topk_idx,
                                 const uint8_t* padding_mask, const void* x,
                                 int32_t* expert_offsets, int32_t* perm_slot, int32_t* inv_perm,
                                 void* x_perm, void* stream);

/*
 * moe_expert_ffn — the routed experts over the permuted rows and the shared
 * experts over all tokens (layers page: inkling_swiglu, InklingSharedExperts).
 * For routed row r of expert e (token t, choice j, weight w = topk_w[t*k+j]):
 *   y_routed[r] = ( w * silu(G[0::2]) * G[1::2] ) @ w_down[e]^T,
 *   G = x_perm[r] @ w_gate_up[e]^T                       (fp32 accumulation)
 * and for shared expert s and token t (weight shared_gamma[t*S+s]) the same
 * with x[t] and ws_*[s] into y_shared[s*T + t].  The activated rows are
 * rounded to dtype (MOE_BF16_F16DOWN: fp16) before the down projection; y
 * rows are written in fp32 (MOE_BF16_F16DOWN: fp16).
 * x_perm may be NULL: the gate_up GEMM then reads row r straight from
 * x[perm_slot[r] / k] (bf16: TMA gathers of 4 rows into the tile), with the
 * same results bit for bit and without the [T*k, H] copy (memory saved:
 * T*k*H elements).  With full tiles this mode is slower than the copy (one
 * TMA instruction per 4 rows and 64 columns instead of one per tile).
 *   perm_slot may be NULL when x_perm is given: the rows are then already in
 *   slot order (row r holds slot r, weight topk_w[r]), as the rows an
 *   expert-parallel rank receives are (moe_ep_dispatch_prep).
 *   x [T,H], x_perm [T*k,H] or NULL, expert_offsets, perm_slot, topk_w [T*k],
 *   shared_gamma [T*S] (NULL iff S == 0), weights as above,
 *   y_routed [T*k, H] out (rows < off[E] written), y_shared [S*T, H] out: fp32
 *   (MOE_BF16_F16DOWN: fp16).
 */
moe_status_t moe_expert_ffn(const moe_layer_desc_t* desc, const void* x, const void* x_perm,
                            const int32_t* expert_offsets, const int32_t* perm_slot,
                            const float* topk_w, const float* shared_gamma,
                            const void* w_gate_up, const void* w_down, const void* ws_gate_up,
                            const void* ws_down, void* y_routed, void* y_shared,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_shared_ffn — the shared experts alone (layers page,
 * InklingSharedExperts.forward(hidden_states, gammas)): for shared expert s
 * and token t,
 *   y_shared[s*T + t] = ( gamma[t,s] * silu(G[0::2]) * G[1::2] ) @ ws_down[s]^T,
 *   G = x[t] @ ws_gate_up[s]^T,
 * with the arithmetic of moe_expert_ffn (bf16: tensor cores, fp32
 * accumulation, activated rows rounded to dtype, y rows fp32).  It serves a
 * rank whose routed experts run elsewhere (expert parallelism).  S >= 1.
 *   x [T,H] dtype, shared_gamma [T,S] fp32, ws_gate_up [S,2I,H],
 *   ws_down [S,H,I], y_shared [S*T,H] out (fp32; MOE_BF16_F16DOWN: fp16);
 *   workspace as moe_workspace_size.
 */
moe_status_t moe_shared_ffn(const moe_layer_desc_t* desc, const void* x, const float* shared_gamma,
                            const void* ws_gate_up, const void* ws_down, void* y_shared,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Number of kernels moe_shared_ffn launches for this layer. */
int32_t moe_shared_ffn_kernel_count(const moe_layer_desc_t* desc);

/*
 * moe_ep_dispatch_prep — the sending side of expert parallelism (layers page:
 * GroupedExperts' expert-parallel sharding; the parallelizer shards
 * InklingMoE.experts over the expert-parallel mesh).  After moe_permute the
 * permuted rows are ordered by global expert, so the rows bound for the rank
 * that owns experts [d*El, (d+1)*El) form one run.  For the R = offsets[E]
 * permuted rows:
 *   row_w[r]         = topk_w[perm_slot[r]]   (the routing weight travels
 *                                              with its row)
 *   expert_counts[e] = offsets[e+1] - offsets[e]
 *   expert_offsets [E+1], perm_slot [T*k] (from moe_permute), topk_w [T*k]
 *   in; row_w [T*k] fp32 out (rows >= R untouched), expert_counts [E] int32
 *   out.  workspace: any buffer of at least 256 bytes whose head is an
 *   initialised status word (a moe_workspace_size() workspace will do); a
 *   slot out of range is recorded there and its row weight is 0.
 */
moe_status_t moe_ep_dispatch_prep(const moe_layer_desc_t* desc, const int32_t* expert_offsets,
                                  const int32_t* perm_slot, const float* topk_w, float* row_w,
                                  int32_t* expert_counts, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * moe_ep_dispatch_p2p — the dispatch of expert parallelism over peer memory
 * (NVLink between the GPUs of a node; same layers-page passages as
 * moe_ep_dispatch_prep).  Rank r's permuted rows go straight from x into
 * the receive buffers of the ranks that own their experts, each with its
 * routing weight: for permuted row i of expert e (offsets[e] <= i <
 * offsets[e+1]), owner d = e / El (El = E / n_ranks) and
 *   dst_x[d][dst_base[e] + i - offsets[e]] = x[perm_slot[i] / k]   (H values)
 *   dst_w[d][dst_base[e] + i - offsets[e]] = topk_w[perm_slot[i]]
 * dst_base[e] is the row of d's receive buffers where this rank's rows of
 * expert e start (the caller computes it from every rank's counts).  No
 * x_perm copy is made (moe_permute may be called with x_perm = NULL).
 *   desc: this rank's layer (T its tokens, E all routed experts);
 *   x [T,H] dtype (16-byte aligned), topk_w [T*k] fp32, perm_slot [T*k],
 *   expert_offsets [E+1] (from moe_permute), dst_base [E] int32 — device;
 *   dst_x, dst_w: device arrays of n_ranks pointers, valid in this process
 *   (this rank's own buffers, or peers' mapped by CUDA IPC), each buffer
 *   dst_rows rows of H dtype values (dst_x) or fp32 (dst_w).  A destination
 *   row outside [0, dst_rows) or a bad slot is recorded in the status word at
 *   the head of `workspace` (>= 256 bytes) and that row is skipped.
 * The kernel only stores; before any rank reads its receive buffers the
 * caller orders every rank's dispatch before that read (an all-reduce over
 * the ranks on the same stream, or a host barrier).  E % n_ranks != 0, or a
 * null or misaligned pointer: MOE_ERR_INVALID_ARG.
 */
moe_status_t moe_ep_dispatch_p2p(const moe_layer_desc_t* desc, const void* x, const float* topk_w,
                                 const int32_t* perm_slot, const int32_t* expert_offsets,
                                 const int32_t* dst_base, int32_t n_ranks, void* const* dst_x,
                                 float* const* dst_w, int64_t dst_rows, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * moe_ep_return_p2p — the return of expert parallelism over peer memory.  A
 * rank's received rows are ordered by local expert el, then by source rank s
 * (run el * n_ranks + s); after moe_expert_ffn its output row i of run j goes
 * back to the source's y rows at the row's place in the source's permuted
 * order:
 *   dst_y[s][src_base[j] + i - run_start[j]] = y_in[i]   (H values)
 *   desc: the layer (H, E, dtype; the rows are fp16 for MOE_BF16_F16DOWN,
 *   else fp32); y_in [rows_in, H]; run_start [E + 1] int32 ascending with
 *   run_start[E] == rows_in, src_base [E] int32 (for run el*n_ranks + s:
 *   source s's expert_offsets[first + el]) — device; dst_y: device array of
 *   n_ranks pointers to buffers of dst_rows rows.  A destination row outside
 *   [0, dst_rows), or run_start[E] != rows_in, is recorded in the status word
 *   and the row (or the call) skipped.  Ordering as for moe_ep_dispatch_p2p.
 */
moe_status_t moe_ep_return_p2p(const moe_layer_desc_t* desc, const void* y_in, int64_t rows_in,
                               const int32_t* run_start, const int32_t* src_base, int32_t n_ranks,
                               void* const* dst_y, int64_t dst_rows, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * moe_combine — InklingMoE.forward recombination:
 *   out[t] = sum_s y_shared[s*T + t] + sum_{j<k, inv_perm[t*k+j] >= 0} y_routed[inv_perm[t*k+j]]
 * summed in fp32 in that fixed order, rounded once to dtype.  y_routed and
 * y_shared are fp32 (MOE_BF16_F16DOWN: fp16); out [T, H] has `dtype`.
 */
moe_status_t moe_combine(const moe_layer_desc_t* desc, const void* y_routed, const void* y_shared,
                         const int32_t* inv_perm, void* out, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * moe_forward — InklingMoE.forward in one call: moe_route, moe_permute,
 * moe_expert_ffn, moe_combine with every intermediate in `workspace`
 * (including the permuted copy x_perm [T*k, H]).  For bf16 layers with
 * shared experts the shared experts' gate_up GEMM runs on a second stream
 * the library keeps for each device (created, with two events, on the first
 * such call; no device memory), forked from `stream` after the router so that
 * it overlaps the permutation and the routed experts' gate_up, and joined
 * back before the down projection, which covers the routed and the shared
 * experts in the same launches.  The call stays asynchronous on `stream` and can be
 * captured in a CUDA graph (the fork and join are captured with it).  Calls
 * from several host threads share that second stream, in call order.
 *   out [T, H] dtype.  topk_w, topk_idx, shared_gamma are optional outputs
 *   (NULL: kept in the workspace).  padding_mask may be NULL.
 */
moe_status_t moe_forward(const moe_layer_desc_t* desc, const void* x, const float* w_router,
                         const float* corr_bias, const void* w_gate_up, const void* w_down,
                         const void* ws_gate_up, const void* ws_down, const uint8_t* padding_mask,
                         void* out, float* topk_w, int32_t* topk_idx, float* shared_gamma,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_selftest_wait_timeout — diagnostic of the stall detection (no
 * counterpart on the pages).  Launches one block that waits, through the
 * same bounded wait every pipeline stage of the grouped GEMM uses, on a
 * barrier nothing arrives on.  After limit_ms (1..10000) the wait gives up
 * and records a timeout in the workspace status word, so that a following
 * moe_read_device_status() returns MOE_ERR_TIMEOUT; the kernel then returns
 * normally and the CUDA context stays usable.
 */
moe_status_t moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_ms,
                                       void* stream);

/* Number of kernels moe_forward launches for this layer (for launch accounting). */
int32_t moe_forward_kernel_count(const moe_layer_desc_t* desc);

/* ------------------------------------------------------------------------
 * The feed-forward block's input norm (InklingRMSNorm, "text" page; the
 * decoder layer's post_attention_layernorm):
 *   out[t, :] = x[t, :] / sqrt(mean_h x[t, h]^2 + eps) * weight
 * over rows of H elements, rounded once (to nearest, ties to even) to
 * `dtype`.  The page states fp32 variance accumulation; this library
 * computes in fp64 and rounds once, so that the rounding (which decides the
 * top-k selection downstream) equals the exact value's rounding except within
 * ~1e-16 of a tie.  weight [H] has `dtype`; eps >= 0 (rms_norm_eps, 1e-6 by
 * default).  x, out [T, H]; out may equal x.  H % 64 == 0.  T = 0 launches
 * nothing.  Asynchronous on `stream`; no workspace.
 * ---------------------------------------------------------------------- */
moe_status_t moe_rmsnorm(int64_t num_tokens, int32_t hidden, moe_dtype_t dtype, float eps,
                         const void* x, const void* weight, void* out, void* stream);

/*
 * moe_forward_prenorm — the block's norm followed by the MoE layer:
 * moe_rmsnorm(x) into the workspace, then moe_forward on it.  Arguments as
 * moe_forward plus norm_weight [H] (dtype) and norm_eps.  The residual add of
 * the decoder block is not part of it.
 */
moe_status_t moe_forward_prenorm(const moe_layer_desc_t* desc, const void* x,
                                 const void* norm_weight, float norm_eps, const float* w_router,
                                 const float* corr_bias, const void* w_gate_up, const void* w_down,
                                 const void* ws_gate_up, const void* ws_down,
                                 const uint8_t* padding_mask, void* out, float* topk_w,
                                 int32_t* topk_idx, float* shared_gamma, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Number of kernels moe_forward_prenorm launches (moe_forward's + 1). */
int32_t moe_forward_prenorm_kernel_count(const moe_layer_desc_t* desc);

/* ------------------------------------------------------------------------
 * The dense feed-forward layer (InklingDenseMLP, "layers" page): the model's
 * decoder layer that has a plain MLP instead of experts (dense_mlp_idx).  It
 * keeps the checkpoint's fused interleaved gate/up projection:
 *   out = global_scale * ( (silu(g) * u) @ w_down^T ),
 *   [g_j, u_j] = rows 2j, 2j+1 of x @ w_gate_up^T
 *   w_gate_up [2I, H] (row 2j = gate_j, row 2j+1 = up_j), w_down [H, I],
 *   x and out [T, H] (leading dims flattened by the caller), all in `dtype`.
 * I is dense_intermediate_size, else intermediate_size (InklingTextConfig).
 * The pages hold global_scale as a parameter of the module without saying
 * where it applies; it scales the output (in exact arithmetic the same as
 * scaling silu(g) * u, which is where the kernels apply it).
 * Same conventions as above; limits: H % 64 == 0, I % 64 == 0, T < 2^26.
 * T = 0 returns MOE_OK without reading any pointer.
 * ---------------------------------------------------------------------- */
typedef struct {
  int64_t num_tokens;    /* T */
  int32_t hidden;        /* H: hidden_size */
  int32_t intermediate;  /* I */
  moe_dtype_t dtype;     /* x, weights, out (MOE_BF16_F16DOWN: w_down fp16) */
  float global_scale;    /* finite */
} moe_dense_desc_t;

/* Workspace bytes for moe_dense_mlp(_prenorm): status word, h [T, I] in dtype,
 * y [T, H] fp32, the normalised input [T, H] in dtype. */
moe_status_t moe_dense_workspace_size(const moe_dense_desc_t* desc, size_t* bytes);

/*
 * moe_dense_mlp — InklingDenseMLP.forward.  bf16 layers run both projections
 * on the tcgen05 tensor cores (bf16 operands, fp32 accumulation; h rounded
 * to bf16, y kept fp32 and rounded once into out); MOE_BF16_F16DOWN layers
 * round h to fp16 and take w_down in fp16 (the down projection's operands);
 * fp32 layers run them in fp32 on the CUDA cores.  Workspace as for the MoE
 * layer: initialise its status word once with moe_workspace_init().
 */
moe_status_t moe_dense_mlp(const moe_dense_desc_t* desc, const void* x, const void* w_gate_up,
                           const void* w_down, void* out, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Number of kernels moe_dense_mlp launches for this layer. */
int32_t moe_dense_kernel_count(const moe_dense_desc_t* desc);

/* moe_dense_mlp_prenorm — moe_rmsnorm(x) into the workspace, then
 * moe_dense_mlp on it (the dense layer's feed-forward block without its
 * residual add).  norm_weight [H] in dtype, norm_eps >= 0. */
moe_status_t moe_dense_mlp_prenorm(const moe_dense_desc_t* desc, const void* x,
                                   const void* norm_weight, float norm_eps, const void* w_gate_up,
                                   const void* w_down, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Number of kernels moe_dense_mlp_prenorm launches (moe_dense_mlp's + 1). */
int32_t moe_dense_prenorm_kernel_count(const moe_dense_desc_t* desc);

/* ------------------------------------------------------------------------
 * moe_convert_bf16_to_f16 — the one-time copy of the down projections'
 * weights for MOE_BF16_F16DOWN layers (no counterpart on the pages: a
 * load-time preparation of the checkpoint's bf16 w_down / ws_down).
 *   n      elements, a multiple of 8 (n = 0 does nothing)
 *   src    bf16 [n], dst fp16 [n] (device, 16-byte aligned, not overlapping):
 *          each value rounded to nearest fp16, which is exact for magnitudes
 *          in [2^-17, 65504] and zero; smaller magnitudes (fp16 subnormals)
 *          change by at most 2^-25
 *   nonfinite  optional device int32 (NULL: none): increased by the number of
 *          elements with no finite fp16 value (magnitude beyond 65504, NaN);
 *          0 means the copy is usable.
 * Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
moe_status_t moe_convert_bf16_to_f16(int64_t n, const void* src, void* dst, int32_t* nonfinite,
                                     void* stream);

const char* moe_status_string(moe_status_t status);
int32_t moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INKLING_MOE_H */
