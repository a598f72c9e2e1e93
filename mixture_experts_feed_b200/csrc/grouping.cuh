// Group and tile bookkeeping of the grouped expert GEMMs.
//
// A launch covers G = E + S groups.  Group g < E is routed expert g: its rows
// are the permuted rows [off[g], off[g+1]) of the routed A operand, its
// weights are slice g of the routed weight tensor, its outputs go to the same
// rows of output 0.  Group E + s is shared expert s: its rows are all T
// tokens, read from A operand 1 starting at row a1_base + s * a1_stride,
// weights are slice s of the shared weight tensor, outputs go to rows
// s * T + t of output 1.
//
// Tiles are numbered group by group.  Inside a group the longer of its two
// tile dimensions is the outer one: with no more m-tiles than n-tiles, tiles
// run n-tile by n-tile and m-tile by m-tile inside (consecutive tiles share
// one weight strip); with more m-tiles than n-tiles, m-tile by m-tile and
// n-tile by n-tile inside (consecutive tiles share one block of rows).  CTAs
// running together then reuse the shared operand from L2, and the group's
// other operand (the n-tile strips, or the row blocks) is the smaller one to
// keep in L2 from one wave of tiles to the next.  A group long in both
// dimensions (more than kBandTiles m-tiles and more than kNarrowStrips
// n-tiles: a dense layer) runs in bands of kBandTiles m-tiles, n-tile by
// n-tile inside a band: a wave covers a near-square block of tiles, the
// band's rows stay in L2 while its strips stream past, and each strip is
// shared by the band's tiles running together.
//
// A group's rows split into mt = ceil(rows / bm) m-tiles of bm rows.  A
// launch covers them in one of three ways (TileSet):
//   kAllTiles  every m-tile, one per tile                       (mt tiles)
//   kPairs     the m-tiles of paired groups two by two, 2*bm rows per tile
//              (ceil(mt / 2) tiles; an odd last pair is half padding)
//   kSingles   the m-tiles of the other groups, one per tile    (mt tiles)
// A group is paired when mt is even, or odd and at least 7: a CTA pair
// moves a third fewer bytes per MMA than one CTA (measured 87% against 73%
// of the bf16 peak per m-tile), which outweighs one padded half-tile from
// 7 m-tiles up, while splitting a group across the two launches would read
// its weights twice.  kPairs and kSingles together cover every row once.
#pragma once

#include <stdint.h>

namespace moe {

struct GroupInfo {
  int src;           // 0 = routed operands, 1 = shared operands
  int b_idx;         // weight slice inside its tensor
  int s;             // shared expert index (src == 1)
  int rows;          // rows in this group
  int64_t a_row0;    // first A row of the group
  int64_t out_row0;  // first output row of the group
};

__device__ __forceinline__ GroupInfo group_info(int g, const int* s_off, int E, int64_t T,
                                                int64_t a1_base, int64_t a1_stride) {
  GroupInfo gi;
  if (g < E) {
    gi.src = 0;
    gi.b_idx = g;
    gi.s = -1;
    gi.a_row0 = s_off[g];
    gi.rows = s_off[g + 1] - s_off[g];
    gi.out_row0 = s_off[g];
  } else {
    const int s = g - E;
    gi.src = 1;
    gi.b_idx = s;
    gi.s = s;
    gi.a_row0 = a1_base + static_cast<int64_t>(s) * a1_stride;
    gi.rows = static_cast<int>(T);
    gi.out_row0 = static_cast<int64_t>(s) * T;
  }
  return gi;
}

enum TileSet { kAllTiles = 0, kPairs = 1, kSingles = 2 };

constexpr int kBandTiles = 8;      // m-tiles per band (tile order, below)
constexpr int kNarrowStrips = 16;  // groups with at most this many n-tiles keep every strip in L2

__host__ __device__ __forceinline__ bool group_paired(int mt) {
  return mt >= 2 && ((mt & 1) == 0 || mt >= 7);
}

__device__ __forceinline__ int tiles_of_rows(int rows, int set, int bm) {
  const int mt = (rows + bm - 1) / bm;
  if (set == kPairs) return group_paired(mt) ? (mt + 1) / 2 : 0;
  if (set == kSingles) return group_paired(mt) ? 0 : mt;
  return mt;
}

// First row (inside its group) of tile m of a group with `rows` rows.
__device__ __forceinline__ int tile_first_row(int m, int rows, int set, int bm) {
  (void)rows;
  return set == kPairs ? m * 2 * bm : m * bm;
}

// Warp 0 of the block fills s_off[0..E] from global memory and
// s_tile[0..G] with the exclusive prefix of per-group tile counts.
// Offsets outside [0, rows_cap] or decreasing are clamped to an empty group
// and reported through `bad` (set to 1).
__device__ inline void build_tile_prefix(const int32_t* __restrict__ offsets, int E, int S,
                                         int64_t T, int set, int bm, int n_tiles, int rows_cap,
                                         int* s_off, int* s_tile, int* bad) {
  const int lane = threadIdx.x & 31;
  if (E == 0) {
    if (lane == 0) s_off[0] = 0;
  } else {
    for (int i = lane; i <= E; i += 32) s_off[i] = offsets[i];
  }
  __syncwarp();
  if (lane == 0 && E > 0) {
    // clamp to a monotone sequence inside [0, rows_cap]
    int prev = 0;
    for (int i = 0; i <= E; ++i) {
      int v = s_off[i];
      if (v < prev || v > rows_cap || (i == 0 && v != 0)) {
        *bad = 1;
        v = v < prev ? prev : (v > rows_cap ? rows_cap : v);
        if (i == 0) v = 0;
      }
      s_off[i] = v;
      prev = v;
    }
  }
  __syncwarp();
  const int G = E + S;
  int carry = 0;
  if (lane == 0) s_tile[0] = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int cnt = 0;
    if (g < G) {
      const int rows = g < E ? (s_off[g + 1] - s_off[g]) : static_cast<int>(T);
      cnt = tiles_of_rows(rows, set, bm) * n_tiles;
    }
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (g < G) s_tile[g + 1] = carry + incl;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
}

// Map a linear tile id to (group, m, n-tile) using the prefix table; the
// tile's first row is tile_first_row(m, rows, set, bm).
__device__ __forceinline__ void decode_tile(int tile, const int* s_tile, int G, const int* s_off,
                                            int E, int64_t T, int set, int bm, int& g, int& m,
                                            int& n) {
  int lo = 0, hi = G - 1;   // find last g with s_tile[g] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tile[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int rows = g < E ? (s_off[g + 1] - s_off[g]) : static_cast<int>(T);
  const int mt = tiles_of_rows(rows, set, bm);
  const int local = tile - s_tile[g];
  const int nt = (s_tile[g + 1] - s_tile[g]) / mt;
  if (mt > kBandTiles && nt > kNarrowStrips) {
    // banded: kBandTiles m-tiles at a time, n-tile by n-tile inside a band
    const int band_tiles = kBandTiles * nt;
    const int band = local / band_tiles;
    const int in_band = local - band * band_tiles;
    const int rows = min(kBandTiles, mt - band * kBandTiles);   // m-tiles in this band
    n = in_band / rows;
    m = band * kBandTiles + (in_band - n * rows);
  } else if (mt > nt) {
    m = local / nt;
    n = local - m * nt;
  } else {
    n = local / mt;
    m = local - n * mt;
  }
}

}  // namespace moe
