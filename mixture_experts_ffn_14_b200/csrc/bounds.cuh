// bounds.cuh — index checks of the MOE_DEBUG_BOUNDS build.
//
// The library's kernels index arrays with values that other kernels computed
// (expert ids, permuted positions, per-expert row ranges). Built with
// -DMOE_DEBUG_BOUNDS they check each such index before the access; a failed
// check records kStatusBounds in the status word (read back through
// moe_device_status) and the access is skipped, so a wrong index shows up as a
// status code instead of a stray read or write. The normal build compiles the
// checks away (kDebugBounds is false).
//
// The predicates are plain host/device functions so that they can also be
// compiled and tested on the host.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define MOE_HD __host__ __device__
#else
#define MOE_HD
#endif

namespace moe {

#ifdef MOE_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// v is an index of an array of n elements.
MOE_HD inline bool index_ok(int64_t v, int64_t n) { return v >= 0 && v < n; }

// The half-open range [first, first + count) lies inside [0, n) (count >= 0;
// an empty range must still start inside [0, n]).
MOE_HD inline bool range_ok(int64_t first, int64_t count, int64_t n) {
  return count >= 0 && first >= 0 && first <= n && count <= n - first;
}

// Per-expert blocks of the permuted rows: counts[e] >= 0, offsets[0] == 0,
// offsets[e + 1] == offsets[e] + counts[e], and the last block ends at `rows`.
MOE_HD inline bool expert_blocks_ok(const int32_t* counts, const int32_t* offsets, int n_experts, int64_t rows) {
  if (offsets[0] != 0) return false;
  for (int e = 0; e < n_experts; ++e) {
    if (counts[e] < 0 || static_cast<int64_t>(offsets[e + 1]) != static_cast<int64_t>(offsets[e]) + counts[e])
      return false;
  }
  return static_cast<int64_t>(offsets[n_experts]) == rows;
}

// A tile of `rows` permuted rows from `row0` and `width` columns from `n0`
// lies inside a [total_rows, n_cols] array.
MOE_HD inline bool tile_ok(int64_t row0, int64_t rows, int64_t total_rows, int64_t n0, int64_t width,
                           int64_t n_cols) {
  return rows >= 1 && range_ok(row0, rows, total_rows) && width >= 1 && range_ok(n0, width, n_cols);
}

}  // namespace moe
