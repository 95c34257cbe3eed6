// Device-side tile list of a grouped GEMM, shared by the tensor-core GEMM
// kernels: every group (expert) g owns rows [offsets[g], offsets[g+1]) of A;
// its row tiles (TILE_M rows, the last one partly empty) times the n_tiles
// column tiles are numbered after those of groups < g, column tile major
// within a group (the row tiles that share a weight tile are adjacent, so the
// CTAs working on them at the same time read that tile from L2 once).
// Groups with no rows own no tile.  The list is derived from the offsets on
// the device, with no host synchronisation.
#pragma once

#include <stdint.h>

namespace moe {

struct TileCoord {
  int g, m_row0, n_tile;
  int m_tile;  // row tile counted over all groups' (padded) row tiles
};

// Warp 0 of a CTA fills s_off[g] = offsets[g] (g <= G) and s_pref[g] = the
// number of the first tile of group g (s_pref[G] = total tiles).
template <int TILE_M>
__device__ __forceinline__ void build_tile_prefix(const int32_t* offsets, int G, int m_total,
                                                  int n_tiles, int lane, int* s_pref, int* s_off) {
  const int per = (G + 31) / 32;
  const int b0 = min(G, lane * per), b1 = min(G, b0 + per);
  int local = 0;
  for (int q = b0; q < b1; ++q) {
    const int o0 = offsets ? offsets[q] : 0;
    const int o1 = offsets ? offsets[q + 1] : m_total;
    s_off[q] = o0;
    const int t = (max(0, o1 - o0) + TILE_M - 1) / TILE_M * n_tiles;
    s_pref[q] = t;
    local += t;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - local;
  for (int q = b0; q < b1; ++q) {
    const int t = s_pref[q];
    s_pref[q] = run;
    run += t;
  }
  if (lane == 31) {
    s_pref[G] = incl;
    s_off[G] = offsets ? offsets[G] : m_total;
  }
}

// Tile number T -> (group, first row, column tile), by binary search over
// the prefix.
template <int TILE_M>
__device__ __forceinline__ TileCoord decode_tile(int T, const int* s_pref, const int* s_off,
                                                 int G, int n_tiles) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= T) lo = mid; else hi = mid - 1;
  }
  TileCoord c;
  c.g = lo;
  const int local = T - s_pref[lo];
  const int mt = (s_off[lo + 1] - s_off[lo] + TILE_M - 1) / TILE_M;
  c.n_tile = local / mt;
  c.m_row0 = s_off[lo] + (local - c.n_tile * mt) * TILE_M;
  c.m_tile = s_pref[lo] / n_tiles + (local - c.n_tile * mt);
  return c;
}

}  // namespace moe
