// Host-compiled check of the token-tile order (mixture_experts_ffn_14_b200/
// csrc/tile_order.cuh): for many expert sizes, group sizes, column-tile and
// split counts, tile_coords maps the tile indices of an expert one to one onto
// its (row tile, column tile, K split) triples, keeps each group's row tiles
// together, and puts the row tile fastest within a group. Exit status 0 = all
// held.
#include <cstdio>
#include <vector>

#include "tile_order.cuh"

int main() {
  using namespace moe;
  int failures = 0;
  long long cases = 0;
  for (int mt = 1; mt <= 70; ++mt) {
    for (int nt = 1; nt <= 26; nt += 5) {
      for (int splits = 1; splits <= 3; ++splits) {
        for (int group : {1, 2, 3, 4, 7, 21, 64}) {
          for (int limit : {1, 6, 32, 1 << 30}) {
            const int g = group_for(mt, group, limit);
            if (g < 1 || g > mt || (mt > limit && g > group)) {
              std::printf("bad group size %d for mt=%d group=%d limit=%d\n", g, mt, group, limit);
              ++failures;
            }
            if (mt > limit) {  // groups as equal as possible: sizes differ by at most one
              const int ng = (mt + g - 1) / g;
              const int last = mt - (ng - 1) * g;
              if (last < 1 || g - last > ng) { std::printf("unbalanced mt=%d g=%d\n", mt, g); ++failures; }
            }
            std::vector<int> seen(mt * nt * splits, 0);
            int prev_mt = -1, prev_nt = -1, prev_ks = -1;
            for (int local = 0; local < mt * nt * splits; ++local) {
              int m, n, k;
              tile_coords(local, mt, nt, g, m, n, k);
              if (m < 0 || m >= mt || n < 0 || n >= nt || k < 0 || k >= splits) {
                std::printf("out of range: mt=%d nt=%d s=%d g=%d local=%d -> %d %d %d\n", mt, nt, splits, g, local, m, n, k);
                ++failures;
                continue;
              }
              seen[(k * nt + n) * mt + m] += 1;
              // within a group and column tile, the row tile advances by one
              if (local > 0 && k == prev_ks && n == prev_nt && m != prev_mt + 1) {
                std::printf("row tile not fastest: mt=%d nt=%d g=%d local=%d\n", mt, nt, g, local);
                ++failures;
              }
              // a tile's group (m / g) never goes back within a K split
              if (local > 0 && k == prev_ks && m / g < prev_mt / g) {
                std::printf("group order broken: mt=%d g=%d local=%d\n", mt, g, local);
                ++failures;
              }
              prev_mt = m; prev_nt = n; prev_ks = k;
            }
            for (int v : seen)
              if (v != 1) { std::printf("not a bijection: mt=%d nt=%d s=%d g=%d\n", mt, nt, splits, g); ++failures; break; }
            ++cases;
          }
        }
      }
    }
  }
  // the group sizes the GEMMs use at the Grok-1 shape: 256-row pair tiles
  if (row_group_size(256, 6144, 64ll << 20) != 21 || row_group_size(256, 32768, 64ll << 20) != 4 ||
      row_group_size(256, 32768, 96ll << 20) != 6 || row_group_size(256, 1ll << 40, 1) != 1) {
    std::printf("row_group_size\n");
    ++failures;
  }
  if (failures == 0) std::printf("tile order ok (%lld cases)\n", cases);
  return failures == 0 ? 0 : 1;
}
