// grouped_tiles.cuh -- the tile schedule shared by the grouped-GEMM kernels.
//
// Groups are the shared experts (dense, m_shared rows each) followed by the routed
// groups (segments of the expert-contiguous slot order, from the device-side offsets).
// A routed group is one expert, or, with expert_mod = n > 0, group g applies expert
// g mod n (rows received from several ranks, grouped by source and then by expert). A
// group of M rows has ceil(M / kTok) token tiles of near-equal size times n_tiles output
// tiles; tiles are numbered group by group, token tiles fastest, so that the CTAs working
// at the same time share each weight tile through L2. The per-group prefix lives in shared
// memory and is built by every CTA from the offsets (no host synchronisation).
#pragma once

#include "kernels.h"

namespace dsmoe {

struct Tile {
  int shared;   // 1: shared-expert group
  int group;    // group index (shared groups first)
  int expert;   // expert index inside its kind
  int row0;     // first token row of the tile
  int m_valid;  // valid token rows in the tile
  int n_blk;    // output tile index
  int kb_n;     // K blocks
};

// Step 1 (all threads of the CTA): tile_start[g + 1] = number of tiles of group g.
template <int kTok>
__device__ __forceinline__ void tile_counts(const GemmArgs& a, int32_t* tile_start, int G) {
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int M, nt;
    if (g < a.n_shared_groups) {
      M = a.m_shared;
      nt = a.n_tiles_shared;
    } else {
      const int e = g - a.n_shared_groups;
      M = a.offsets[e + 1] - a.offsets[e];
      nt = a.n_tiles_routed;
    }
    M = max(M, 0);
    tile_start[g + 1] = ((M + kTok - 1) / kTok) * nt;
  }
  if (threadIdx.x == 0) tile_start[0] = 0;
}

// Step 2 (one whole warp, after a CTA barrier): inclusive prefix over tile_start[1..G].
__device__ __forceinline__ void tile_scan(int32_t* tile_start, int G, int lane) {
  int carry = 0;
  for (int b0 = 1; b0 <= G; b0 += 32) {
    const int i = b0 + lane;
    int v = (i <= G) ? tile_start[i] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (i <= G) tile_start[i] = v + carry;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
}

template <int kTok>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, const int32_t* tile_start, int G, int tile) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // last group whose first tile is <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  Tile t;
  t.group = lo;
  int M, base;
  if (lo < a.n_shared_groups) {
    t.shared = 1;
    t.expert = lo;
    M = a.m_shared;
    base = 0;
    t.kb_n = a.kb_shared;
  } else {
    t.shared = 0;
    const int gi = lo - a.n_shared_groups;  // routed group: its segment of the offsets
    t.expert = a.expert_mod > 0 ? gi % a.expert_mod : gi;  // its weights
    base = a.offsets[gi];
    M = a.offsets[gi + 1] - base;
    t.kb_n = a.kb_routed;
  }
  const int mt = (M + kTok - 1) / kTok;
  const int local = tile - tile_start[lo];
  const int m_blk = local % mt;
  t.n_blk = local / mt;
  // The group's rows are split evenly over its mt token tiles in 16-row granules (tile
  // sizes differ by at most 16), not into full tiles and one ragged remainder: the CTAs
  // sharing a weight tile then run at the same MMA rate and stay close enough in K for
  // the second reader to find the weights in L2. The MMA work is the same, since N is
  // the tile's row count rounded up to 16 either way.
  const int gr = (M + 15) >> 4, q = gr / mt, rem = gr - q * mt;
  const int g0 = m_blk * q + min(m_blk, rem);
  t.row0 = base + g0 * 16;
  t.m_valid = min((q + (m_blk < rem ? 1 : 0)) * 16, M - g0 * 16);
  return t;
}

}  // namespace dsmoe
