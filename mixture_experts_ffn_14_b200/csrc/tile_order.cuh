// tile_order.cuh — order of the tiles of one expert in the token-tile GEMMs.
//
// An expert's tiles are (row tile mt, column tile nt, K split ks). Consecutive
// tile ids run at about the same time on different SMs (they are handed out in
// order), so the order decides what they share in L2:
//   - row tile fastest: the concurrently running tiles read one weight tile
//     (read once from DRAM) and different activation row tiles;
//   - but when an expert holds many row tiles, all of its activation rows are
//     live at once (a 16384-row expert: 201 MB of X for the gate/up GEMM, 1 GB
//     of H for the down GEMM), more than L2 holds, and they are fetched from
//     DRAM again for every column tile.
// So the row tiles of an expert whose activation block is larger than L2 go
// in groups of at most `group` (sized by the caller so that a group's rows fit
// in L2): within a K split, group 0's row tiles for every column tile (row tile
// fastest), then group 1's, and so on. The weight tiles are then read once per
// group instead of once, the activation rows once instead of once per column
// tile. Splitting costs a re-read of the expert's weights per extra group, so
// an expert whose block fits stays one group (the plain row-tile-fastest
// order): at the Grok-1 shape the down projection's weights (402 MB per
// expert) are larger than a prefill expert's intermediate rows (64-80 MB).
#pragma once

#if defined(__CUDACC__)
#define MOE_TO_HD __host__ __device__
#else
#define MOE_TO_HD
#endif

namespace moe {

// local: tile index within the expert (0 .. mt_count * nt_count * splits - 1).
MOE_TO_HD inline void tile_coords(int local, int mt_count, int nt_count, int group, int& mt, int& nt, int& ks) {
  const int per_ks = mt_count * nt_count;
  ks = local / per_ks;
  int r = local - ks * per_ks;
  const int g = r / (group * nt_count);  // the full groups come first, the last may be smaller
  const int g0 = g * group;
  const int gsize = mt_count - g0 < group ? mt_count - g0 : group;
  r -= g0 * nt_count;
  mt = g0 + r % gsize;
  nt = r / gsize;
}

// Group size for an expert of mt_count row tiles: all of them when
// mt_count <= limit, else the fewest groups of at most `group` row tiles, made
// as equal as possible (so no group is a lone remainder that re-reads the
// weights for one row tile).
MOE_TO_HD inline int group_for(int mt_count, int group, int limit) {
  if (mt_count <= limit) return mt_count > 0 ? mt_count : 1;
  const int ng = (mt_count + group - 1) / group;
  return (mt_count + ng - 1) / ng;
}

// Row tiles whose activation rows (tile_rows x k_elems 16-bit values each)
// take at most `budget_bytes`; at least 1. The caller uses it for the group
// size and for the largest expert that stays one group.
MOE_TO_HD inline int row_group_size(long long tile_rows, long long k_elems, long long budget_bytes) {
  const long long per = tile_rows * k_elems * 2;
  const long long g = per > 0 ? budget_bytes / per : 1;
  return g < 1 ? 1 : (g > (1 << 20) ? (1 << 20) : static_cast<int>(g));
}

}  // namespace moe
