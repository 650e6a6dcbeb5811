// Host-compiled check of the index predicates of the MOE_DEBUG_BOUNDS build
// (mixture_experts_ffn_14_b200/csrc/bounds.cuh): in-range and out-of-range
// indices, ranges and per-expert row blocks. Exit status 0 = all held.
#include <cstdint>
#include <cstdio>

#include "bounds.cuh"

static int failures = 0;
#define CHECK(cond)                                               \
  do {                                                            \
    if (!(cond)) {                                                \
      std::printf("check failed, line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                 \
    }                                                             \
  } while (0)

int main() {
  using namespace moe;
  // index_ok: [0, n)
  CHECK(index_ok(0, 1));
  CHECK(index_ok(8191, 8192));
  CHECK(!index_ok(8192, 8192));
  CHECK(!index_ok(-1, 8192));
  CHECK(!index_ok(0, 0));
  CHECK(index_ok((int64_t(1) << 33) - 1, int64_t(1) << 33));  // indices past 2^31
  CHECK(!index_ok(int64_t(1) << 33, int64_t(1) << 33));

  // range_ok: [first, first + count) inside [0, n)
  CHECK(range_ok(0, 128, 128));
  CHECK(range_ok(100, 28, 128));
  CHECK(!range_ok(100, 29, 128));
  CHECK(range_ok(128, 0, 128));         // empty range at the end
  CHECK(!range_ok(129, 0, 128));
  CHECK(!range_ok(-1, 1, 128));
  CHECK(!range_ok(0, -1, 128));
  CHECK(!range_ok(int64_t(1) << 62, int64_t(1) << 62, int64_t(1) << 62));  // no overflow in the sum

  // expert_blocks_ok: counts and offsets of 8 experts over 2T rows
  int32_t counts[8] = {3, 0, 5, 1, 0, 0, 2, 1};
  int32_t offsets[9] = {0, 3, 3, 8, 9, 9, 9, 11, 12};
  CHECK(expert_blocks_ok(counts, offsets, 8, 12));
  CHECK(!expert_blocks_ok(counts, offsets, 8, 13));  // blocks do not end at the row count
  offsets[4] = 10;                                   // block 3 and 4 inconsistent
  CHECK(!expert_blocks_ok(counts, offsets, 8, 12));
  offsets[4] = 9;
  counts[1] = -1;                                    // negative count
  offsets[2] = 2;
  offsets[3] = 7;
  offsets[4] = 8;
  offsets[5] = offsets[6] = offsets[7] = 8;
  offsets[7] = 10;
  offsets[8] = 11;
  CHECK(!expert_blocks_ok(counts, offsets, 8, 11));
  int32_t c2[8] = {1, 1, 1, 1, 1, 1, 1, 1};
  int32_t o2[9] = {1, 2, 3, 4, 5, 6, 7, 8, 9};       // does not start at 0
  CHECK(!expert_blocks_ok(c2, o2, 8, 9));

  // tile_ok: rows of a tile and its column block inside [total_rows, n_cols]
  CHECK(tile_ok(0, 128, 8192, 0, 256, 6144));
  CHECK(tile_ok(8064, 128, 8192, 5888, 256, 6144));
  CHECK(!tile_ok(8065, 128, 8192, 0, 256, 6144));   // rows past the end
  CHECK(!tile_ok(0, 0, 8192, 0, 256, 6144));        // empty tile
  CHECK(!tile_ok(0, 128, 8192, 6000, 256, 6144));   // columns past the end
  CHECK(!tile_ok(-128, 128, 8192, 0, 256, 6144));
  CHECK(!tile_ok(0, 128, 8192, -256, 256, 6144));

  if (failures == 0) std::printf("bounds predicates ok\n");
  return failures == 0 ? 0 : 1;
}
