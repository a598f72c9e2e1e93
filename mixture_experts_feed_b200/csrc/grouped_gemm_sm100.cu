// Grouped GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel computes, for every group of rows (a routed expert or
// a shared expert, see grouping.cuh), D = A_rows @ W_g^T with bf16 operands
// and an fp32 accumulator in tensor memory, then runs a fused epilogue:
//   kGateUp: the accumulator columns interleave gate and up channels
//            ([g0, u0, g1, u1, ...], the fused gate_up_proj layout of the
//            Inkling layers page, inkling_swiglu); the epilogue writes
//            h = w * silu(g) * u in bf16, or in fp16 when the down
//            projection runs in fp16, w the row's routing weight (routed
//            rows: topk_w of the row's slot; shared rows: the token's gamma,
//            or one uniform weight when no gamma is given: the dense layer,
//            run as a single shared group, passes its global_scale).
//   kDown:   bf16 x bf16, or fp16 x fp16 (fp16 h against an fp16 copy of the
//            weights); the epilogue writes D in fp32, or fp16 with fp16
//            operands, and the recombination sums the rows in fp32 and
//            rounds the layer output once (bf16 rows would put a correctly
//            rounded pipeline beyond the 2e-2 x RMS bound).
//   kRouter: router logits z = x @ Wr^T, the fp32 router bank split exactly
//            into three bf16 parts (W = W0 + W1 + W2) so that every product
//            is exact.  The tensor-core accumulator loses about one fp32 ulp
//            of its own magnitude per MMA step (measured: 5.7e-5 in z over a
//            3 x 6144 chain), so each accumulation chain is kept to two
//            64-deep K blocks: the MMA writes a fresh chain sum, and the
//            epilogue warps add the chain sums in fp32 registers with
//            round-to-nearest adds.  fp32 logits out.  One group (all T
//            tokens), N = E + S, 160-column tiles (E + S = 129 in one tile,
//            257 in two).  The parts run chunk by chunk over K (part 2, 1, 0
//            of one 1024-deep chunk, then the next), so the three reads of
//            an x block come from L2.
//
// The expert modes run on CTA pairs (clusters of two SMs, tcgen05
// cta_group::2): a pair computes a 256-row x 256-column tile with M=256
// MMAs; each CTA loads its own 128 A rows and half of the 256 B rows, so the
// bytes each SM pulls per MMA drop by a third against one-SM 128 x 256 tiles
// and six pipeline stages fit in shared memory.  The router runs one CTA per
// tile (M=128).
//
// Roles (192 threads per CTA, one CTA per SM):
//   warp 0      TMA producer: per stage, this CTA's A tile [128 rows x 64 K]
//               and its B rows [BN/2 (pairs) or BN rows x 64 K], 128-byte
//               swizzle; pair loads signal the rank-0 CTA's barrier.  Lane 0
//               waits on the stages and issues the loads; when the routed A
//               rows are gathered straight from x (kGateUp without x_perm),
//               each lane issues one tile::gather4 of 4 of the 128 rows.
//   warp 1      TMEM allocator and (rank-0 CTA only) MMA issuer, one thread:
//               4 x tcgen05.mma K16 per stage into one of two accumulators
//               (2 x BN TMEM columns in each CTA; the router keeps three).
//   warps 2..5  epilogue: tcgen05.ld this CTA's accumulator rows (warp w
//               reads TMEM lanes 32*(w%4) .. +31), fused math, global stores.
// The two accumulators let the epilogue of one tile (or, for kRouter, one K
// chain) overlap the MMAs of the next.  Tiles go to the CTAs (CTA pairs) in
// a fixed order, or, when the launch is given a tile counter (the gate_up
// pair launch with long K), as the rank-0 producer draws them, handed to
// the other roles through a tile queue in shared memory.  All waits are bounded
// (sm100_ptx.cuh); on a timeout every role stops, the status word records it
// and TMEM is released.  No TMA load uses cluster multicast.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "grouping.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace sm100 {

constexpr int BM = 128;          // A rows per CTA
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;
// kRouter: K blocks per tensor-core accumulation chain (128-deep chains)
constexpr int ROUTER_CHAIN = 2;
// kRouter: K blocks per chunk.  The three weight parts run chunk by chunk
// (part 2, 1, 0 over one chunk of K, then the next chunk), so each CTA reads
// a 128 x 1024 block of x three times while it is still in L2 instead of
// streaming x from HBM once per part.
constexpr int ROUTER_CHUNK = 16;

// kRouter: the K block and weight part of step kt of a CTA's 3 * k_blocks
// steps (chunk-major; a last, shorter chunk when k_blocks is not a multiple
// of ROUTER_CHUNK).
__device__ __forceinline__ void router_step(int kt, int k_blocks, int& kb, int& part) {
  const int full = k_blocks / ROUTER_CHUNK;
  const int c = kt / (3 * ROUTER_CHUNK);
  const int size = c < full ? ROUTER_CHUNK : k_blocks - full * ROUTER_CHUNK;
  const int r = kt - c * 3 * ROUTER_CHUNK;
  part = 2 - r / size;
  kb = c * ROUTER_CHUNK + r % size;
}

enum Mode { kGateUp = 0, kDown = 1, kRouter = 2 };

template <int MODE, bool PAIR_> struct Tile {
  static constexpr bool PAIR = PAIR_;                       // CTA-pair (M=256) MMAs
  // which m-tiles of each group the launch covers (grouping.cuh)
  static constexpr int SET = PAIR ? kPairs : (MODE == kRouter ? kAllTiles : kSingles);
  static constexpr int BN = MODE == kRouter ? 160 : 256;    // MMA N = accumulator columns
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;         // B rows one CTA loads
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int B_BOX = MODE == kRouter ? BN : 128;  // rows per B tensor-map box
  static constexpr int B_LOADS = B_ROWS / B_BOX;            // boxes per stage
  // Pipeline stages: one stage = this CTA's A tile followed by its B rows,
  // stages back to back in one ring of RING_BYTES.  Single-CTA expert
  // launches with n-tiles of at most 128 columns (half the B bytes a stage)
  // run NARROW_STAGES stages in the same ring, so that as many weight bytes
  // stay in flight when the launch only streams weights.
  static constexpr int STAGES = PAIR ? 6 : 4;               // stages of full-width tiles
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int NARROW_STAGES = (!PAIR && MODE != kRouter) ? RING_BYTES / (A_BYTES + B_BYTES / 2) : STAGES;
  // Single-CTA expert launches whose tiles hold at most 32 rows (few
  // tokens) keep 32-row A tiles, so that more stages of weights fit the
  // ring: up to RING_BYTES / (4 KB + B_BYTES / 2) with narrow n-tiles.
  static constexpr bool SHORT_OK = !PAIR && MODE != kRouter;
  static constexpr int SHORT_A_BYTES = 32 * BK * 2;
  static constexpr int MAX_STAGES = SHORT_OK ? RING_BYTES / (SHORT_A_BYTES + B_BYTES / 2)
                                             : (NARROW_STAGES > STAGES ? NARROW_STAGES : STAGES);
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;         // rows per tile
  // accumulators: two (the epilogue of one tile overlaps the next tile's
  // MMAs); the router's 160-column accumulation chains keep three, so that
  // the MMAs run a chain further ahead of the epilogue that sums them.  The
  // allocation is rounded up to a power of two.
  static constexpr int NACC = MODE == kRouter ? 3 : 2;
  static constexpr uint32_t TMEM_COLS = NACC * BN <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, BN);
};

struct alignas(64) GemmParams {
  CUtensorMap tmA[2];   // A operand of routed (0) and shared (1) groups: 2-D [rows, K]
  CUtensorMap tmB[2];   // weights of routed (0) and shared (1) groups: 3-D [G][N][K]
  CUtensorMap tmY[2];   // kDown: output rows of routed (0) and shared (1) groups: fp32, box
                        // 32 rows x 32 columns, or fp16, box 32 x 64 (128 bytes a row either way)
  const int32_t* offsets;     // [E+1]
  const int32_t* perm_slot;   // [rows] slot of each permuted row (kGateUp weights)
  const float* topk_w;        // [T*k]
  const float* gamma;         // [T*S], or null: every shared row gets uniform_w
  float uniform_w;
  void* out[2];               // output of routed (0) and shared (1) groups
  int32_t* status;
  int64_t T;
  int64_t a1_base, a1_stride; // shared group s reads A rows from a1_base + s*a1_stride
  int E, S, K, N;
  int ld_out;                 // output row length in elements
  int rows_cap;               // rows of the routed A operand (bound of offsets)
  int ksplit;                 // kRouter, kDown: K-range splits (each writes its own partial)
  int bn;                     // single-CTA expert launches: n-tile width (32..256, multiple of 32)
  int gather_k;               // kGateUp: > 0 = routed A rows are gathered from x (tmA[0] over
                              // [T, H], box one row high): row r reads x[perm_slot[r] / gather_k]
  int f16;                    // kGateUp: h written in fp16; kDown: A (h) and B (weights) fp16
  int y_f16;                  // kDown: output rows in fp16 (tmY boxes 32 rows x 64 columns)
  int64_t split_stride;       // kRouter: elements between partial outputs
  int* tile_counter;          // tiles drawn from this counter (zero at launch), or null: the
                              // fixed order (tile unit, unit + units, ...)
  int a_rows;                 // single-CTA expert launches: A rows a stage holds, 128, or 32
                              // when no tile has more rows (the A maps' boxes are that high)
};

// Per epilogue warp, a 32 x 32 fp32 staging tile (row stride 36 floats:
// 16-byte aligned, and each quarter-warp's 16-byte accesses hit distinct banks).
constexpr int STAGE_LD = 36;
// 5120 bytes a warp (the padded tile needs 4608): every warp's region starts
// on a 1024-byte boundary, as a 128-byte-swizzled TMA box requires
constexpr int STAGE_WARP_BYTES = 5120;

// Tile queue of the dynamic schedule: slots holding the tiles the producer
// drew, read by the CTA's other roles (and, in a pair, by the other CTA).
constexpr int TQ = 8;

template <int MODE, bool PAIR> struct SmemLayout {
  static constexpr int MAX_STAGES = Tile<MODE, PAIR>::MAX_STAGES;
  static constexpr int kRing = 0;                                   // the stage ring
  static constexpr int kStage = Tile<MODE, PAIR>::RING_BYTES;       // 4 x STAGE_WARP_BYTES
  static constexpr int kBars = kStage + 4 * STAGE_WARP_BYTES;
  // full[MAX_STAGES], empty[MAX_STAGES], tfull[3], tempty[3], drain, qfull[TQ], qempty[TQ]
  static constexpr int kNumBars = 2 * MAX_STAGES + 7 + 2 * TQ;
  static constexpr int kMisc = kBars + kNumBars * 8;   // tmem base, abort, bad
  static constexpr int kQueue = kMisc + 16;            // the tile queue's slots
  static constexpr int kTables = kQueue + 4 * TQ;
};

template <int MODE, bool PAIR>
__host__ __device__ inline int smem_bytes(int E, int S) {
  return 1024 /* alignment slack */ + SmemLayout<MODE, PAIR>::kTables + 4 * ((E + 1) + (E + S + 1));
}

// Write one warp's 32 rows x 32 fp32 columns through the staging tile so that
// each store instruction covers 4 whole 128-byte row segments.
__device__ __forceinline__ void store_rows_f32(float* st, const uint32_t (&v)[32], int lane,
                                               float* out, int64_t row0, int rows_left,
                                               int64_t ld, int col0) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(st + lane * STAGE_LD + 4 * q) =
        make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int sub_row = lane >> 3;          // 0..3
  const int sub_col = (lane & 7) * 4;     // 0..28
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int rr = it * 4 + sub_row;      // row inside the warp's 32
    const float4 val = *reinterpret_cast<const float4*>(st + rr * STAGE_LD + sub_col);
    if (rr < rows_left)
      *reinterpret_cast<float4*>(out + (row0 + rr) * ld + col0 + sub_col) = val;
  }
  __syncwarp();
}

// The same for 32 rows x 64 fp16 columns (32 packed words a lane: 128 bytes
// of its row), staged with a 36-word row stride.
__device__ __forceinline__ void store_rows_f16(uint32_t* st, const uint32_t (&w)[32], int lane,
                                               uint16_t* out, int64_t row0, int rows_left,
                                               int64_t ld, int col0) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(st + lane * STAGE_LD + 4 * q) =
        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  __syncwarp();
  const int sub_row = lane >> 3;          // 0..3
  const int sub_col = (lane & 7) * 4;     // word offset 0..28 (8 fp16 each 4 words)
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int rr = it * 4 + sub_row;
    const uint4 val = *reinterpret_cast<const uint4*>(st + rr * STAGE_LD + sub_col);
    if (rr < rows_left)
      *reinterpret_cast<uint4*>(out + (row0 + rr) * ld + col0 + 2 * sub_col) = val;
  }
  __syncwarp();
}

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using TL = Tile<MODE, PAIR>;
  using SL = SmemLayout<MODE, PAIR>;
  constexpr int BN = TL::BN;
  constexpr int NACC = TL::NACC;
  constexpr int STAGES = TL::MAX_STAGES;   // barrier arrays; the ring runs `stages` of them
  constexpr int SET = TL::SET;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem + SL::kRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL::kBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 3;
  uint64_t* drain = bars + 2 * STAGES + 6;
  uint64_t* qfull = bars + 2 * STAGES + 7;
  uint64_t* qempty = qfull + TQ;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SL::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SL::kMisc + 4);
  int* s_bad = reinterpret_cast<int*>(smem + SL::kMisc + 8);
  int* s_tq = reinterpret_cast<int*>(smem + SL::kQueue);
  int* s_off = reinterpret_cast<int*>(smem + SL::kTables);
  int* s_tile = s_off + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;     // 0 = the pair's MMA issuer
  const bool leader = rank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int G = p.E + p.S;
  // kRouter and kDown fold their K splits into the n-tile index: nv = n * ksplit + ks
  const int ksplit = MODE == kGateUp ? 1 : p.ksplit;
  // n-tile width: the MMA's full N, except single-CTA expert launches, which
  // may use narrower tiles (more tiles for layers with few rows)
  const int bn = (PAIR || MODE == kRouter) ? BN : p.bn;
  // the stage ring: narrow single-CTA tiles (bn <= 128) take half the B bytes
  // a stage, and 32-row A tiles a quarter of the A bytes; the ring then
  // holds more stages.  With 32-row A tiles the M=128 MMA also reads the 96
  // rows after them (the start of the stage's own B rows, loaded with them):
  // those accumulator rows lie past every group and are never stored.
  const bool narrow = TL::NARROW_STAGES != TL::STAGES && bn <= 128;
  const int a_stage_bytes = (TL::SHORT_OK && p.a_rows == 32) ? TL::SHORT_A_BYTES : A_BYTES;
  const int stage_bytes = a_stage_bytes + (narrow ? TL::B_BYTES / 2 : TL::B_BYTES);
  const int stages = min(STAGES, TL::RING_BYTES / stage_bytes);
  auto stage_a = [&](int st) { return ring + st * stage_bytes; };                  // A tile of a stage
  auto stage_b = [&](int st) { return ring + st * stage_bytes + a_stage_bytes; };  // its B rows
  const int n_tiles = (p.N + bn - 1) / bn * ksplit;
  const int k_blocks = p.K / BK;                               // per weight part
  const int k_total = MODE == kRouter ? 3 * k_blocks : k_blocks;
  // K-block range [kt_begin(ks), kt_begin(ks + 1)) of split ks
  auto kt_begin = [&](int ks) { return static_cast<int>(static_cast<int64_t>(k_total) * ks / ksplit); };

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], 1);
      }
      for (int i = 0; i < 3; ++i) {
        mbar_init(&tfull[i], 1);
        mbar_init(&tempty[i], PAIR ? 8 : 4);   // one arrive per epilogue warp (of both CTAs)
      }
      mbar_init(drain, 1);
      for (int i = 0; i < TQ; ++i) {
        mbar_init(&qfull[i], 1);
        // one arrive per reader of a slot: the MMA issuer and the 4 epilogue
        // warps, and in a pair also the other CTA's producer and epilogue warps
        mbar_init(&qempty[i], PAIR ? 10 : 5);
      }
      *s_abort = 0;
      *s_bad = 0;
      fence_mbar_init();
      fence_proxy_async_smem();
      prefetch_tmap(&p.tmA[0]);
      prefetch_tmap(&p.tmA[1]);
      prefetch_tmap(&p.tmB[0]);
      prefetch_tmap(&p.tmB[1]);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(s_tmem, TL::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s_tmem, TL::TMEM_COLS);
      tmem_relinquish();
    }
  } else if (warp == 2) {
    pdl_wait();
    build_tile_prefix(p.offsets, p.E, p.S, p.T, SET, BM, n_tiles, p.rows_cap, s_off, s_tile, s_bad);
  }
  // The setup above (barriers, tensor memory, tensor-map prefetch) may run
  // while the previous kernel on the stream finishes; every global access
  // below comes after it has completed.
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();   // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();

  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = s_tile[G];
  if (threadIdx.x == 0 && *s_bad) record_status(p.status, DEV_BAD_ROW);

  // The tile schedule.  Every role of a CTA (and both CTAs of a pair) walks
  // the same sequence of tiles; -1 ends it.  With a tile counter the pair's
  // rank-0 producer draws each next tile with an atomic add, so clusters
  // that start late or run slow tiles take fewer of them and all of them
  // stay on nearby tiles, and passes it through the tile queue (slot
  // seq % TQ): qfull[slot] completes when a tile is written (in a pair, into
  // both CTAs' slots), qempty[slot] when every reader has taken it.  Without
  // a counter tiles go out in the fixed order unit, unit + units, ...
  const bool dyn = MODE != kRouter && p.tile_counter != nullptr;
  auto static_tile = [&](int seq) {
    const int64_t t = static_cast<int64_t>(unit) + static_cast<int64_t>(seq) * units;
    return t < total_tiles ? static_cast<int>(t) : -1;
  };
  // rank-0 producer (lane 0): publish `tile` as tile `seq` of the sequence
  auto publish_tile = [&](int seq, int tile) -> bool {
    const int slot = seq % TQ;
    if (!mbar_wait_cluster(&qempty[slot], ((seq / TQ) & 1) ^ 1u, s_abort, p.status)) return false;
    s_tq[slot] = tile;
    mbar_arrive(&qfull[slot]);
    if (PAIR) {
      st_shared_cluster_u32(mapa_shared(&s_tq[slot], 1), static_cast<uint32_t>(tile));
      mbar_arrive_cluster(mapa_shared(&qfull[slot], 1));
    }
    return true;
  };
  // any other reader (one thread): take tile `seq` from the queue and free
  // its slot (the value is then in a register)
  auto take_tile = [&](int seq, int& tile) -> bool {
    const int slot = seq % TQ;
    const uint32_t parity = (seq / TQ) & 1;
    if (!(PAIR ? mbar_wait_cluster(&qfull[slot], parity, s_abort, p.status)
               : mbar_wait(&qfull[slot], parity, s_abort, p.status)))
      return false;
    tile = *reinterpret_cast<volatile int*>(&s_tq[slot]);
    if (tile >= 0) {
      if (!PAIR || leader) mbar_arrive(&qempty[slot]);
      else mbar_arrive_cluster(mapa_shared(&qempty[slot], 0));
    }
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int last_parity[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) last_parity[i] = -1;
    // rank-0 producer, lane 0: tiles are published one tile ahead and drawn
    // two ahead, so that neither the atomic nor the hand-over to the other
    // CTA sits between the loads of two tiles.  cur = tile seq (published),
    // nxt = tile seq + 1 (its atomic in flight during tile seq - 1).
    auto drawn = [&](int t) { return t >= 0 && t < total_tiles ? t : -1; };
    int cur = -1, nxt = -1;
    int prologue_ok = 1;
    if (dyn && leader) {   // warp-uniform
      if (lane == 0) {
        cur = drawn(atomicAdd(p.tile_counter, 1));
        prologue_ok = publish_tile(0, cur) ? 1 : 0;
        if (cur >= 0) nxt = atomicAdd(p.tile_counter, 1);
      }
      prologue_ok = __shfl_sync(0xffffffffu, prologue_ok, 0);
    }
    for (int seq = 0; prologue_ok; ++seq) {
      int tile = -1;
      if (!dyn) {
        tile = static_tile(seq);
      } else {
        int got = 1;
        if (lane == 0) {
          if (leader) {
            tile = cur;
            if (tile >= 0) {
              const int t1 = drawn(nxt);
              if (!publish_tile(seq + 1, t1)) {
                got = 0;
              } else {
                cur = t1;
                if (t1 >= 0) nxt = atomicAdd(p.tile_counter, 1);
              }
            }
          } else {
            got = take_tile(seq, tile) ? 1 : 0;
          }
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (!got) break;
      }
      if (tile < 0) break;
      int g, m, nv;
      decode_tile(tile, s_tile, G, s_off, p.E, p.T, SET, BM, g, m, nv);
      const int n = nv / ksplit, ks = nv - n * ksplit;
      const GroupInfo gi = group_info(g, s_off, p.E, p.T, p.a1_base, p.a1_stride);
      const void* tmA = &p.tmA[gi.src];
      const void* tmB = &p.tmB[gi.src];
      const int a_row = static_cast<int>(gi.a_row0) + tile_first_row(m, gi.rows, SET, BM) +
                        static_cast<int>(rank) * BM;
      // pairs: this CTA's half of the tile's (possibly narrowed) N range
      const int n_pad = (min(bn, p.N - n * bn) + 31) & ~31;
      const int b_row = n * bn + (PAIR ? static_cast<int>(rank) * (n_pad >> 1) : 0);
      // single-CTA expert tiles load only the 128-row boxes the tile covers
      const int b_loads = (PAIR || MODE == kRouter) ? TL::B_LOADS : (n_pad + TL::B_BOX - 1) / TL::B_BOX;
      // gathered A rows: lane l loads rows 4l..4l+3 of this CTA's 128, from
      // token perm_slot[row] / gather_k.  Lanes whose 4 rows all lie past
      // the group load nothing (those rows of the tile keep stale data: their
      // results are never stored); a lane's rows past the group read token 0.
      const bool gather = MODE == kGateUp && p.gather_k > 0 && gi.src == 0;
      const int tile_row0 = tile_first_row(m, gi.rows, SET, BM);   // tile's first row in the group
      auto gathered_bytes = [&](int r) {      // A bytes the gathers of CTA r bring per stage
        const int rows_r = min(BM, max(0, gi.rows - tile_row0 - r * BM));
        return ((rows_r + 3) / 4) * 4 * BK * 2;
      };
      int tok[4] = {0, 0, 0, 0};
      const int first = tile_row0 + static_cast<int>(rank) * BM + 4 * lane;   // row inside the group
      const bool lane_gathers = gather && first < gi.rows;
      const int a_bytes = gather ? (PAIR ? gathered_bytes(0) + gathered_bytes(1) : gathered_bytes(0))
                                 : (PAIR ? 2 * A_BYTES : a_stage_bytes);
      if (gather) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (first + q < gi.rows) {
            const int slot = p.perm_slot[gi.a_row0 + first + q];
            if (slot >= 0 && slot < p.rows_cap) {
              tok[q] = slot / p.gather_k;
            } else {
              record_status(p.status, DEV_BAD_ROW);
            }
          }
        }
      }
      bool ok = true;
      for (int kt = kt_begin(ks); kt < kt_begin(ks + 1); ++kt) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty[stage], phase ^ 1u, s_abort, p.status) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        // router: per chunk of K, part 2 (smallest) first, then 1, then 0
        int kb = kt, slice = gi.b_idx;
        if (MODE == kRouter) router_step(kt, k_blocks, kb, slice);
        uint8_t* a_dst = stage_a(stage);
        if (PAIR) {
          // both CTAs' bytes complete on the rank-0 CTA's barrier
          const uint32_t bar0 = mapa_shared(&full[stage], 0);
          if (lane == 0) {
            if (leader) mbar_arrive_expect_tx(&full[stage], a_bytes + 2 * TL::B_BYTES);
            if (!gather) tma_load_2d_pair(a_dst, tmA, bar0, kb * BK, a_row);
            tma_load_3d_pair(stage_b(stage), tmB, bar0, kb * BK, b_row, slice);
          }
          if (lane_gathers)
            tma_gather4_pair(a_dst + lane * 4 * BK * 2, tmA, bar0, kb * BK, tok[0], tok[1], tok[2],
                             tok[3]);
        } else {
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], a_bytes + b_loads * (TL::B_BOX * BK * 2));
            if (!gather) tma_load_2d(a_dst, tmA, &full[stage], kb * BK, a_row);
            for (int i = 0; i < b_loads; ++i)
              tma_load_3d(stage_b(stage) + i * (TL::B_BOX * BK * 2), tmB, &full[stage],
                          kb * BK, b_row + i * TL::B_BOX, slice);
          }
          if (lane_gathers)
            tma_gather4(a_dst + lane * 4 * BK * 2, tmA, &full[stage], kb * BK, tok[0], tok[1],
                        tok[2], tok[3]);
        }
        last_parity[stage] = static_cast<int>(phase);
        if (++stage == stages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    // no more loads from this CTA: the next kernel on the stream may be
    // scheduled (its CTAs take an SM once one of this launch's CTAs exits)
    pdl_trigger();
    // Wait (bounded) until the last load issued on every stage has landed,
    // so that no copy still writes shared memory when the block exits.  A
    // pair's loads all complete on the rank-0 CTA's barriers; the other CTA
    // is covered by the cluster barrier at the end.
    const uint64_t t0 = globaltimer_ns();
    for (int i = 0; i < STAGES && leader && lane == 0; ++i) {
      if (last_parity[i] < 0) continue;
      while (!mbar_try_wait(&full[i], static_cast<uint32_t>(last_parity[i]))) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) { record_status(p.status, DEV_WAIT_TIMEOUT); break; }
      }
    }
    __syncwarp();
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;   // accumulator hand-offs so far (tiles, or K blocks for kRouter)
    bool ok = true;
    for (int seq = 0; ok; ++seq) {
      int tile = -1;
      if (!dyn) tile = static_tile(seq);
      else if (!take_tile(seq, tile)) { ok = false; break; }
      if (tile < 0) break;
      int g, m, nv;
      decode_tile(tile, s_tile, G, s_off, p.E, p.T, SET, BM, g, m, nv);
      const int n = nv / ksplit, ks = nv - n * ksplit;
      // a narrow or ragged last n-tile runs a narrower MMA (N multiple of 32)
      const int n_here = min(bn, p.N - n * bn);
      uint32_t idesc = n_here >= BN ? TL::IDESC : idesc_bf16_f32(TL::TILE_M, (n_here + 31) & ~31);
      if (MODE == kDown && p.f16) idesc = idesc_as_f16(idesc);   // fp16 h and fp16 weights
      if (MODE != kRouter) {
        const int acc = it % NACC;
        if (!mbar_wait(&tempty[acc], ((it / NACC) & 1) ^ 1u, s_abort, p.status)) { ok = false; break; }
        tc_fence_after();
      }
      const int kb0 = kt_begin(ks), kb1 = kt_begin(ks + 1);
      for (int kb = kb0; kb < kb1; ++kb) {
        const int acc = it % NACC;
        // router: a hand-off at the start of every chain of ROUTER_CHAIN K blocks
        const bool chain_start = MODE == kRouter && (kb - kb0) % ROUTER_CHAIN == 0;
        const bool chain_end = MODE == kRouter && ((kb - kb0) % ROUTER_CHAIN == ROUTER_CHAIN - 1 || kb + 1 == kb1);
        if (chain_start) {
          if (!mbar_wait(&tempty[acc], ((it / NACC) & 1) ^ 1u, s_abort, p.status)) { ok = false; break; }
          tc_fence_after();
        }
        if (!mbar_wait(&full[stage], phase, s_abort, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const uint64_t adesc = smem_desc_kmajor_sw128(smem_u32(stage_a(stage)));
        const uint64_t bdesc = smem_desc_kmajor_sw128(smem_u32(stage_b(stage)));
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // +32 bytes per K=16 step inside the 128-byte swizzle atom
          // router: a fresh sum per chain; experts: accumulate over the tile
          const bool accumulate = MODE == kRouter ? (!chain_start || kk != 0) : (((kb - kb0) | kk) != 0);
          if (PAIR)
            mma_bf16_ss_pair(d_tmem, adesc + static_cast<uint64_t>(2 * kk),
                             bdesc + static_cast<uint64_t>(2 * kk), idesc, accumulate ? 1u : 0u);
          else
            mma_bf16_ss(d_tmem, adesc + static_cast<uint64_t>(2 * kk),
                        bdesc + static_cast<uint64_t>(2 * kk), idesc, accumulate ? 1u : 0u);
        }
        if (PAIR) mma_commit_pair(&empty[stage], 0x3);   // frees the stage in both CTAs
        else mma_commit(&empty[stage]);
        if (++stage == stages) { stage = 0; phase ^= 1u; }
        if (chain_end) {
          mma_commit(&tfull[acc]);
          ++it;
        }
      }
      if (!ok) break;
      if (MODE != kRouter) {
        if (PAIR) mma_commit_pair(&tfull[it % NACC], 0x3);
        else mma_commit(&tfull[it % NACC]);
        ++it;
      }
    }
    // Every MMA this thread issued must be complete before TMEM is freed.
    if (PAIR) mma_commit_pair(drain, 0x1);
    else mma_commit(drain);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) { record_status(p.status, DEV_WAIT_TIMEOUT); break; }
    }
  } else if (warp >= 2) {
    // --------------------------------------------------------- epilogue
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const int row_in_tile = quarter * 32 + lane;
    float* st = reinterpret_cast<float*>(smem + SL::kStage) + (warp - 2) * (STAGE_WARP_BYTES / 4);
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int it = 0;
    bool ok = true;
    bool h_overflow = false;   // an activated value beyond the fp16 range
    for (int seq = 0; ok; ++seq) {
      int tile = -1;
      if (!dyn) {
        tile = static_tile(seq);
      } else {
        int got = 1;
        if (lane == 0) got = take_tile(seq, tile) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (!got) { ok = false; break; }
      }
      if (tile < 0) break;
      int g, m, nv;
      decode_tile(tile, s_tile, G, s_off, p.E, p.T, SET, BM, g, m, nv);
      const int n = nv / ksplit, ks = nv - n * ksplit;
      const GroupInfo gi = group_info(g, s_off, p.E, p.T, p.a1_base, p.a1_stride);
      const int row0 = tile_first_row(m, gi.rows, SET, BM) + static_cast<int>(rank) * BM;   // this CTA's first row
      const int r = row0 + row_in_tile;            // row inside the group
      const bool valid = r < gi.rows;
      const int64_t out_row = gi.out_row0 + r;
      const int rows_left = gi.rows - (row0 + quarter * 32);   // rows of this warp's 32

      if (MODE == kRouter) {
        // Sum the per-K-block accumulators in fp32 registers (round to nearest).
        float run[BN];
#pragma unroll
        for (int i = 0; i < BN; ++i) run[i] = 0.0f;
        const int kb0 = kt_begin(ks), kb1 = kt_begin(ks + 1);
        const int chains = (kb1 - kb0 + ROUTER_CHAIN - 1) / ROUTER_CHAIN;
        for (int ch = 0; ch < chains; ++ch) {
          const int acc = it % NACC;
          if (!mbar_wait(&tfull[acc], (it / NACC) & 1, s_abort, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < BN / 32; c += 2) {
            if (n * BN + c * 32 < p.N) {            // warp-uniform
              uint32_t v[32], v2[32];
              tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(acc * BN + c * 32), v);
              const bool second = c + 1 < BN / 32 && n * BN + (c + 1) * 32 < p.N;
              if (second) tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(acc * BN + (c + 1) * 32), v2);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) run[c * 32 + i] += __uint_as_float(v[i]);
              if (second) {
#pragma unroll
                for (int i = 0; i < 32; ++i) run[(c + 1) * 32 + i] += __uint_as_float(v2[i]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
          ++it;
        }
        if (!ok) break;
        float* out = static_cast<float*>(p.out[gi.src]) + ks * p.split_stride;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          const int col0 = n * BN + c * 32;
          if (col0 < p.N) {
            uint32_t v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(run[c * 32 + i]);
            store_rows_f32(st, v, lane, out, gi.out_row0 + row0 + quarter * 32, rows_left,
                           p.ld_out, col0);
          }
        }
        continue;
      }

      const int acc = it % NACC;
      if (!mbar_wait(&tfull[acc], (it / NACC) & 1, s_abort, p.status)) break;
      tc_fence_after();
      float w = 1.0f;
      if (MODE == kGateUp && valid) {
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
      }
      const uint32_t t_row = t_lane + static_cast<uint32_t>(acc * BN);
      const int n_here = min(bn, p.N - n * bn);
      if (MODE == kDown && p.y_f16) {
        // fp16 output rows: two 32-column chunks make one 128-byte row
        // segment (n_here is a multiple of 64: H % 64 == 0); each 32-row slab
        // goes through the swizzled staging box and one TMA store, as below
#pragma unroll 1
        for (int c = 0; c < BN / 32; c += 2) {
          const int col0 = n * bn + c * 32;
          if (c * 32 >= n_here) break;             // warp-uniform
          uint32_t v[32], v2[32], pk[32];
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), v);
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 1) * 32), v2);
          tmem_ld_wait();
          bool ovf = false;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[i] = pack_f16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]), ovf);
            pk[16 + i] = pack_f16x2(__uint_as_float(v2[2 * i]), __uint_as_float(v2[2 * i + 1]), ovf);
          }
          // only rows of the group count: rows past its end hold whatever the
          // A operand's rows beyond the group held, and are never stored
          if (valid && ovf) h_overflow = true;
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
          if (rows_left >= 32) {
            uint8_t* box = reinterpret_cast<uint8_t*>(st);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&p.tmY[gi.src], box, col0,
                           static_cast<int32_t>(gi.out_row0 + row0 + quarter * 32));
              bulk_commit_group();
            }
          } else {
            store_rows_f16(reinterpret_cast<uint32_t*>(st), pk, lane,
                           static_cast<uint16_t*>(p.out[gi.src]), gi.out_row0 + row0 + quarter * 32,
                           rows_left, p.ld_out, col0);
          }
        }
      } else {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = n * bn + c * 32;
        if (c * 32 >= n_here) break;               // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), v);
        tmem_ld_wait();
        if (MODE == kGateUp) {
          if (!valid) continue;
          uint32_t packed[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g0 = __uint_as_float(v[4 * i + 0]);
            const float u0 = __uint_as_float(v[4 * i + 1]);
            const float g1 = __uint_as_float(v[4 * i + 2]);
            const float u1 = __uint_as_float(v[4 * i + 3]);
            // silu(g) = g / (1 + e^-g) with the fast division (2 ulp): the
            // product is rounded to bf16 or fp16 right after
            const float h0 = w * __fdividef(g0, 1.0f + __expf(-g0)) * u0;
            const float h1 = w * __fdividef(g1, 1.0f + __expf(-g1)) * u1;
            // fp16 down projections: h rounded to fp16 (8x finer than bf16)
            packed[i] = p.f16 ? pack_f16x2(h0, h1, h_overflow) : pack_bf16x2(h0, h1);
          }
          uint16_t* out = static_cast<uint16_t*>(p.out[gi.src]);   // bf16 or fp16 bits
          uint4* dst = reinterpret_cast<uint4*>(out + out_row * p.ld_out + col0 / 2);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        } else {
          if (rows_left >= 32) {
            // a full 32-row slab: the 32 x 32 fp32 chunk goes through a
            // 128-byte-swizzled staging box (chunk j of row r at 16-byte slot
            // j ^ (r & 7): conflict-free) and one TMA store; only the buffer
            // reuse waits, for the previous store to have read it.  K split
            // ks writes the partial rows at row offset ks * T.
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            uint8_t* box = reinterpret_cast<uint8_t*>(st);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&p.tmY[gi.src], box, col0,
                           static_cast<int32_t>(ks * p.T + gi.out_row0 + row0 + quarter * 32));
              bulk_commit_group();
            }
          } else {
            // the group's last rows: coalesced stores of the valid rows only
            // (a box would write into the next group's rows)
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            store_rows_f32(st, v, lane, static_cast<float*>(p.out[gi.src]) + ks * p.split_stride,
                           gi.out_row0 + row0 + quarter * 32, rows_left, p.ld_out, col0);
          }
        }
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));   // the issuer's barrier
        else mbar_arrive(&tempty[acc]);
      }
      ++it;
    }
    if (MODE != kRouter && __any_sync(0xffffffffu, h_overflow) && lane == 0)
      record_status(p.status, DEV_F16_OVERFLOW);
    // the warp's TMA stores complete before the block (and its shared memory) goes
    if (MODE == kDown && lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();   // no MMA or signal of the pair is still in flight
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, TL::TMEM_COLS);
    else tmem_dealloc(tmem_base, TL::TMEM_COLS);
  }
}

// ------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D bf16 map over [rows, K] (K contiguous), box [box_rows, BK], 128B
// swizzle: BM rows for tile loads, one row for tile::gather4.
static bool encode_a(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows = BM,
                     bool f16 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 map over [rows, H] (H contiguous), box [32 rows, 32 columns],
// 128B swizzle: the down projection's output rows, written by TMA stores.
static bool encode_y(CUtensorMap* m, void* base, int64_t rows, int H, bool f16 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * (f16 ? 2 : 4)};
  cuuint32_t box[2] = {f16 ? 64u : 32u, 32};   // 128 bytes a row
  cuuint32_t estr[2] = {1, 1};
  return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base,
             dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 (or fp16) map over [G][N][K] (K contiguous), box [1][bn][BK], 128B swizzle.
static bool encode_b(CUtensorMap* m, const void* base, int G, int N, int K, int bn,
                     bool f16 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(G)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2,
                           static_cast<cuuint64_t>(K) * 2 * static_cast<cuuint64_t>(N)};
  cuuint32_t box[3] = {BK, static_cast<cuuint32_t>(bn), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, bool PAIR>
static cudaError_t launch_mode(const GemmParams& p, int sms, cudaStream_t stream) {
  const int smem = smem_bytes<MODE, PAIR>(p.E, p.S);
  // the attribute is per device; calls from several host threads may set it
  // concurrently (same value), devices past 64 set it on every launch
  static std::atomic<int> configured_smem[64];
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64;
  if (!cached || configured_smem[dev].load(std::memory_order_relaxed) < smem) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, PAIR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (cached) {
      int seen = configured_smem[dev].load(std::memory_order_relaxed);
      while (seen < smem && !configured_smem[dev].compare_exchange_weak(seen, smem)) {
      }
    }
  }
  // programmatic stream serialisation (see pdl_wait), and CTA pairs as
  // clusters of two
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(PAIR ? (sms & ~1) : sms), 1, 1);   // whole pairs
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, PAIR>, p);
}

}  // namespace sm100

// gate_up: A0 = x_perm [T*k, H], or, with x_perm null, x [T, H] gathered
// row by row through perm_slot; A1 = x [T, H]; out0 = h rows [0, T*k),
// out1 = h rows T*k + s*T + t.  down: A0 = A1 = h [T*k + S*T, I];
// out0 = y_routed, out1 = y_shared.
cudaError_t launch_expert_ffn_bf16(const Layer& L, const void* x, const void* x_perm,
                                   const int32_t* offsets, const int32_t* perm_slot,
                                   const float* topk_w, const float* gamma, const void* w_gate_up,
                                   const void* w_down, const void* ws_gate_up,
                                   const void* ws_down, void* h, void* y_routed, void* y_shared,
                                   int32_t* status, int num_sms, cudaStream_t stream,
                                   bool* map_error, const FfnTiling& tiling) {
  using namespace sm100;
  // B maps: box of 128 rows = the half of a 256-row n-tile one CTA of a pair
  // loads; the single-CTA odd-tile launch loads both halves (two boxes)
  constexpr int BROWS = Tile<kGateUp, true>::B_BOX;
  *map_error = false;
  const int64_t Rk = L.T * L.k;                 // routed row capacity
  const int64_t Rh = Rk + static_cast<int64_t>(L.S) * L.T;
  __nv_bfloat16* hb = static_cast<__nv_bfloat16*>(h);
  // paired groups on CTA pairs, the rest on single CTAs (grouping.cuh); with
  // T <= 128 every group has one m-tile and the pair launch is skipped
  // (E == 0, the dense layer: the host knows the one group's m-tiles and
  // launches only the kind of CTA that has tiles)
  const bool pairs = L.T > BM && (L.E > 0 || group_paired(static_cast<int>((L.T + BM - 1) / BM)));
  const bool singles = L.E > 0 || !pairs;
  // tiling.part: both projections, or one of them (a caller that splits the
  // two around a join of streams)
  const bool do_gate_up = tiling.part != 2, do_down = tiling.part != 1;
  // The gate_up pair launch with long K (H >= 4096) draws its tiles from a
  // counter (the dynamic schedule of the kernel): its clusters then stay on
  // a narrow window of consecutive tiles, whose A rows and weight strips L2
  // holds, where the fixed order lets slow clusters fall behind and widen
  // it (measured on a B200 at T=8192, H=6144, E=128, k=8, I=2048: 4.5
  // instead of 9.8 GB read from DRAM by that launch).  Short-K launches keep
  // the fixed order, which costs less per tile.  The counter lives in the
  // status region (a call of the shared
  // groups alone, E == 0, takes the next one, so that it can run on another
  // stream beside a call of the routed groups) and is zeroed here.
  int* gate_up_counter = nullptr;
  if (status != nullptr && pairs && L.H >= 4096 && do_gate_up) {
    gate_up_counter = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(status) + kTileCounterOffset) +
                      (L.E == 0 ? 1 : 0);
    const cudaError_t e = cudaMemsetAsync(gate_up_counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
  }

  // ---------------- gate_up: [rows, H] x [2I, H]^T -> SwiGLU -> h [rows, I]
  // With no routed rows (E == 0: the dense layer) the routed maps are never
  // read; they are encoded over the shared operands so that every map is valid.
  const bool routed = L.E > 0 && Rk > 0;
  const bool gather = routed && x_perm == nullptr;
  // With T <= 32 no group has more rows than T (a token takes an expert at
  // most once), so the single-CTA launches keep 32-row A tiles
  const int a_rows = L.T <= 32 ? 32 : BM;
  GemmParams g{};
  bool ok = (gather ? encode_a(&g.tmA[0], x, L.T, L.H, 1)
                    : encode_a(&g.tmA[0], routed ? x_perm : x, routed ? Rk : L.T, L.H, a_rows)) &&
            encode_a(&g.tmA[1], x, L.T, L.H, a_rows);
  if (ok && L.E > 0) ok = encode_b(&g.tmB[0], w_gate_up, L.E, 2 * L.I, L.H, BROWS);
  if (ok && L.S > 0) ok = encode_b(&g.tmB[1], ws_gate_up, L.S, 2 * L.I, L.H, BROWS);
  if (L.E == 0) g.tmB[0] = g.tmB[1];
  if (L.S == 0) g.tmB[1] = g.tmB[0];
  if (!ok) { *map_error = true; return cudaErrorInvalidValue; }
  g.offsets = offsets; g.perm_slot = perm_slot; g.topk_w = topk_w; g.gamma = gamma;
  g.uniform_w = L.global_scale;
  g.out[0] = hb;
  g.out[1] = hb + Rk * L.I;
  g.status = status;
  g.T = L.T; g.a1_base = 0; g.a1_stride = 0;
  g.E = L.E; g.S = L.S; g.K = L.H; g.N = 2 * L.I; g.ld_out = L.I;
  g.rows_cap = static_cast<int>(Rk);
  g.ksplit = 1;
  g.bn = tiling.gate_up_bn;
  g.gather_k = gather ? L.k : 0;
  g.f16 = L.down_f16 ? 1 : 0;   // h in fp16 for fp16 down projections
  g.a_rows = a_rows;
  cudaError_t e = cudaSuccess;
  if (!do_gate_up) {
    // the activated rows are already in h
  } else if (tiling.gate_up_ksplit > 1) {
    // The dense layer with few tokens: gate_up as a plain GEMM with its K
    // split (the kDown mode's fp32 partial stores: split s at rows s * T of
    // gate_up_part [ks * T, 2I]), then the SwiGLU over the partials.  More
    // tiles than the n-tiles alone give fill the SMs in whole waves.
    const int ks = tiling.gate_up_ksplit;
    if (L.E != 0 || L.S != 1 || pairs || tiling.gate_up_part == nullptr) return cudaErrorInvalidValue;
    GemmParams q{};
    ok = encode_a(&q.tmA[0], x, L.T, L.H, a_rows) &&
         encode_b(&q.tmB[0], ws_gate_up, 1, 2 * L.I, L.H, BROWS) &&
         encode_y(&q.tmY[0], tiling.gate_up_part, L.T * static_cast<int64_t>(ks), 2 * L.I);
    if (!ok) { *map_error = true; return cudaErrorInvalidValue; }
    q.tmA[1] = q.tmA[0];
    q.tmB[1] = q.tmB[0];
    q.tmY[1] = q.tmY[0];
    q.out[0] = q.out[1] = tiling.gate_up_part;
    q.status = status;
    q.T = L.T; q.a1_base = 0; q.a1_stride = L.T;
    q.E = 0; q.S = 1; q.K = L.H; q.N = 2 * L.I; q.ld_out = 2 * L.I;
    q.rows_cap = 0;
    q.ksplit = ks;
    q.split_stride = L.T * static_cast<int64_t>(2 * L.I);
    q.bn = 256;
    q.a_rows = a_rows;
    e = launch_mode<kDown, false>(q, num_sms, stream);
    if (e == cudaSuccess)
      e = launch_swiglu_partials(tiling.gate_up_part, ks, L.T, L.I, L.global_scale, L.down_f16,
                                 h, status, num_sms, stream);
  } else {
    g.tile_counter = gate_up_counter;
    e = pairs ? launch_mode<kGateUp, true>(g, num_sms, stream) : cudaSuccess;
    g.tile_counter = nullptr;
    if (e == cudaSuccess && singles) e = launch_mode<kGateUp, false>(g, num_sms, stream);
  }
  if (e != cudaSuccess || !do_down) return e;

  // ---------------- down: h [rows, I] x [H, I]^T -> y [rows, H] (fp32)
  GemmParams d{};
  const bool f16 = L.down_f16;   // h and the down weights in fp16
  ok = encode_a(&d.tmA[0], h, Rh, L.I, a_rows, f16);
  if (ok && L.E > 0) ok = encode_b(&d.tmB[0], w_down, L.E, L.H, L.I, BROWS, f16);
  d.tmA[1] = d.tmA[0];
  if (ok && L.S > 0) ok = encode_b(&d.tmB[1], ws_down, L.S, L.H, L.I, BROWS, f16);
  if (L.E == 0) d.tmB[0] = d.tmB[1];
  if (L.S == 0) d.tmB[1] = d.tmB[0];
  // output maps: routed rows [T*k, H]; shared rows [S*T, H], or one partial
  // [T, H] per K split when the down projection splits K (the dense layer)
  const int64_t shared_rows = L.T * static_cast<int64_t>(L.S > tiling.down_ksplit ? L.S : tiling.down_ksplit);
  const bool y_f16 = L.y_f16 && tiling.down_ksplit == 1;   // K-split partials stay fp32
  if (ok && L.S > 0) ok = encode_y(&d.tmY[1], y_shared, shared_rows, L.H, y_f16);
  if (ok && routed) ok = encode_y(&d.tmY[0], y_routed, Rk, L.H, y_f16);
  if (!routed) d.tmY[0] = d.tmY[1];
  if (L.S == 0) d.tmY[1] = d.tmY[0];
  if (!ok) { *map_error = true; return cudaErrorInvalidValue; }
  d.offsets = offsets; d.perm_slot = perm_slot; d.topk_w = topk_w; d.gamma = gamma;
  d.uniform_w = L.global_scale;
  d.out[0] = y_routed;
  d.out[1] = y_shared;
  d.status = status;
  d.T = L.T; d.a1_base = Rk; d.a1_stride = L.T;
  d.E = L.E; d.S = L.S; d.K = L.I; d.N = L.H; d.ld_out = L.H;
  d.rows_cap = static_cast<int>(Rk);
  d.ksplit = tiling.down_ksplit;
  d.split_stride = L.T * static_cast<int64_t>(L.H);   // partial rows of the shared groups
  d.bn = 256;
  d.f16 = f16 ? 1 : 0;
  d.y_f16 = y_f16 ? 1 : 0;
  d.a_rows = a_rows;
  e = pairs ? launch_mode<kDown, true>(d, num_sms, stream) : cudaSuccess;
  if (e == cudaSuccess && singles) e = launch_mode<kDown, false>(d, num_sms, stream);
  return e;
}

// Router logits on the tensor cores: ksplit partial sums z_s[T, ld_z] (fp32,
// ld_z = E+S rounded up to 32, consecutive in `logits`) with
// sum_s z_s = x [T, H] @ (W0 + W1 + W2)^T, W_p the bf16 parts [3][E+S][H].
cudaError_t launch_router_logits_sm100(const Layer& L, const void* x, const void* w_parts,
                                       float* logits, int ld_z, int ksplit, int32_t* status,
                                       int num_sms, cudaStream_t stream, bool* map_error) {
  using namespace sm100;
  *map_error = false;
  const int NE = L.E + L.S;
  GemmParams r{};
  const bool ok = encode_a(&r.tmA[0], x, L.T, L.H) &&
                  encode_b(&r.tmB[0], w_parts, 3, NE, L.H, Tile<kRouter, false>::B_BOX);
  if (!ok) { *map_error = true; return cudaErrorInvalidValue; }
  r.tmA[1] = r.tmA[0];
  r.tmB[1] = r.tmB[0];
  r.offsets = nullptr; r.perm_slot = nullptr; r.topk_w = nullptr; r.gamma = nullptr;
  r.out[0] = logits;
  r.out[1] = logits;
  r.status = status;
  r.T = L.T; r.a1_base = 0; r.a1_stride = 0;
  r.E = 0; r.S = 1;                 // one group: all T tokens
  r.K = L.H; r.N = NE; r.ld_out = ld_z;
  r.rows_cap = 0;
  r.ksplit = ksplit;
  r.split_stride = L.T * static_cast<int64_t>(ld_z);
  r.bn = Tile<kRouter, false>::BN;
  return launch_mode<kRouter, false>(r, num_sms, stream);
}


}  // namespace moe
