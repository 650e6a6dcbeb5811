// moe_internal.cuh — declarations shared by the library's translation units:
// workspace layout, device status bits and kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/moe.h"
#include "bounds.cuh"

namespace moe {

constexpr int kE = 8;              // experts (this version)
constexpr int kK = 2;              // experts per token
constexpr int kRouteTokens = 32;   // tokens per router / dispatch CTA
constexpr int64_t kTallMinT = 512;  // bf16 gate/up under MOE_PATH_AUTO: 256-row tiles from this many tokens

// Device status word bits (set with atomicOr; 0 = no failure recorded).
enum : uint32_t {
  kStatusProducerTimeout = 1u << 0,
  kStatusMmaTimeout = 1u << 1,
  kStatusEpilogueTimeout = 1u << 2,
  kStatusConvertTimeout = 1u << 3,
  kStatusSelftestTimeout = 1u << 4,
  // int8-weight path: an activation or GeGLU intermediate outside the fp16
  // range (|v| > 65504 rounds to infinity) in the conversion to fp16.
  kStatusFp16Range = 1u << 5,
  // MOE_DEBUG_BOUNDS builds: an index outside its array was caught and the
  // access skipped.
  kStatusBounds = 1u << 6,
};

// Byte offsets of the regions of one call's workspace (each 256-aligned).
struct WorkspaceLayout {
  size_t status, arrivals, combine_count, idx, gates, hist, hist_pre, logits_part, counts, offsets, perm_token, perm_slot,
      slot_pos, gate_perm;
  size_t xp, h, y, total;
  int64_t nblk;      // router / dispatch CTAs
  int32_t splits;    // split-K factor of the down projection
  int32_t router_slices;  // d slices of the router grid
  bool weight_stream;  // down projection in the weight-stream form (and gate/up unless gateup_tt)
  // bf16 weights, automatic path, weight-stream batch: the gate/up GEMM runs
  // 128-row token tiles on single CTAs, the down projection weight-stream tiles.
  bool gateup_tt;
  bool tile_path;    // gate/up in token tiles (bf16 / int8 weights): row gather possible
};

// Host: workspace layout for a call (valid arguments assumed).
WorkspaceLayout plan_workspace(int64_t T, int64_t d, int64_t f, moe_dtype_t dtype, moe_path_t path,
                               int32_t down_splits, bool h_external);

// Host: which kernel family a call uses.
bool use_weight_stream(int64_t T, moe_path_t path, moe_dtype_t dtype);
int32_t choose_down_splits(int64_t T, int64_t d, int64_t f, int32_t requested);

// ---- launchers (return cudaSuccess or the launch error) --------------------

// Router: grid of (token blocks, d slices). With slices > 1 the CTAs store
// partial logits in `partial` [slices, T, E] and count their arrivals per token
// block in `arrivals` [nblk] (zero on entry); the last one finishes the block.
int32_t router_slices(int64_t T, int64_t d, moe_dtype_t dtype);
cudaError_t launch_router(moe_dtype_t dtype, const void* x, const float* w_router, const float* bias, int64_t T,
                          int64_t d, int32_t renormalize, int32_t slices, float* partial, int32_t* arrivals,
                          int32_t* idx, float* gates, int32_t* hist, cudaStream_t s);

// Dispatch. With more than kDispatchSumBlocks router blocks a one-CTA scan of
// the block histograms runs first, into hist_pre [nblk * E + E] (prefixes, then
// totals); with fewer, each dispatch CTA sums the histograms it needs itself.
constexpr int64_t kDispatchSumBlocks = 1024;
cudaError_t launch_dispatch(moe_dtype_t dtype, const void* x, int64_t T, int64_t d, int64_t nblk,
                            const int32_t* idx, const float* gates, const int32_t* hist, int32_t* hist_pre,
                            int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                            int32_t* slot_pos, float* gate_perm, void* xp, uint32_t* status,
                            cudaStream_t s);  // xp == nullptr: no row copy

// Small batches (1 <= T <= 128, d <= 65536, with the permuted copy, and a
// device on which a 16-CTA cluster fits): router and dispatch in one cluster
// launch; same outputs as the two launches above (idx, gates, counts, offsets,
// perm_token, perm_slot, slot_pos, gate_perm, xp).
bool small_route_dispatch(int64_t T, int64_t d, const void* xp);
cudaError_t launch_route_dispatch_small(moe_dtype_t dtype, const void* x, const float* w_router, const float* bias,
                                        int64_t T, int64_t d, int32_t renormalize, int32_t* idx, float* gates,
                                        int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                                        int32_t* slot_pos, float* gate_perm, void* xp, uint32_t* status,
                                        cudaStream_t s);

// out[t] = residual[t] + norm(y0 + y1); residual and norm_weight may be NULL.
// Expert-parallel pieces: counts of n local experts -> the kE-slot counts and
// offsets the GEMM kernels read (zero rows for the other slots), plus 1.0 gates
// for rows without one; the fixed-order sum of split-K partials; a row gather.
cudaError_t launch_local_schedule(const int32_t* counts_in, int32_t n, int32_t* counts, int32_t* offsets,
                                  float* ones, int64_t n_ones, cudaStream_t s);
cudaError_t launch_sum_splits(const float* part, int64_t split_stride, int32_t splits, int64_t n, float* y,
                              cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, int64_t src_rows, const int32_t* index, int64_t n,
                               int64_t row_bytes, void* dst, uint32_t* status, cudaStream_t s);

cudaError_t launch_combine(moe_dtype_t dtype, const float* y, int64_t split_stride, int32_t splits,
                           const int32_t* slot_pos, int64_t T, int64_t d, const void* residual,
                           const float* norm_weight, float norm_eps, void* out, uint32_t* status, cudaStream_t s);

// fp32 (SIMT) grouped expert GEMMs.
cudaError_t launch_f32_gateup(const float* xp, const float* wg, const float* wu, const int32_t* counts,
                              const int32_t* offsets, int64_t T, int64_t d, int64_t f, int32_t act,
                              float* h, uint32_t* status, cudaStream_t s);
cudaError_t launch_f32_down(const float* h, const float* wd, const int32_t* counts, const int32_t* offsets,
                            const float* gate_perm, int64_t T, int64_t d, int64_t f, float* y, uint32_t* status,
                            cudaStream_t s);

// tcgen05 grouped expert GEMMs (bf16 or int8 weights).
struct TcGemmArgs {
  const void* x;            // [rows, K] bf16 activations (Xp or H), rows = 2T; x [x_rows, K] with row_token
  const int32_t* row_token; // GATEUP token tiles: token of each permuted row (A rows gathered from x), or nullptr
  int64_t x_rows;           // rows of x when row_token is set (T)
  const void* w0;           // [E, K, N] gate (GATEUP) or down (DOWN) weights, bf16 or int8
  const void* w1;           // [E, K, N] up weights (GATEUP) or nullptr
  const __nv_bfloat16* s0;  // int8: [E, N] scales of w0, else nullptr
  const __nv_bfloat16* s1;  // int8: [E, N] scales of w1, else nullptr
  const int32_t* counts;
  const int32_t* offsets;
  const float* gate_perm;   // DOWN: gate of each permuted row
  void* out;                // GATEUP: H bf16 [rows, N]; DOWN: Y fp32 [splits, rows, N]
  int64_t rows;             // 2T
  int32_t K, N;
  int32_t splits;           // DOWN split-K factor (1 for GATEUP)
  int32_t act;              // moe_activation_t
  bool int8_weights;
  bool weight_stream;
  int32_t select;           // 0: always run; 1 / 2: run only if the pair / single token-tile form is preferred
  int32_t* tile_counter;    // pair form: zeroed int that hands out tiles in order, or nullptr (static order)
  int32_t* tile_counter_single;  // single-CTA token tiles: the same, for that form's launch
  uint32_t* status;
  int32_t n_experts;        // experts in the weight arrays (0 = kE); experts past it have no rows
  bool short_tiles;         // weight-stream: tiles of at most 64 tokens, deeper weight ring
  bool tall_tiles;          // bf16 GATEUP token tiles: 256-row tiles on single CTAs (int8 always uses them)
  // DOWN token tiles: the combine in the epilogue (out[t] = sum of the two
  // gate-scaled rows of token t, in fixed order). combine_count == nullptr:
  // the epilogue only writes Y and a separate combine kernel runs.
  const int32_t* perm_token;  // [rows] token of each permuted row
  const int32_t* slot_pos;    // [T, 2] permuted row of each (token, slot)
  int32_t* combine_count;     // [T, N/256] arrivals per (token, column tile), zero on entry
  void* combine_out;          // [T, N] bf16 sublayer output
  const void* residual;       // [T, N] bf16 added to the output, or nullptr
};
cudaError_t launch_tc_gateup(const TcGemmArgs& a, cudaStream_t s);
cudaError_t launch_tc_down(const TcGemmArgs& a, cudaStream_t s);
// Token-tile form on CTA pairs (cta_group::2); `weight_stream` must be false.
cudaError_t launch_tc_gateup_pair(const TcGemmArgs& a, cudaStream_t s);
cudaError_t launch_tc_down_pair(const TcGemmArgs& a, cudaStream_t s);

// Host: encode a TMA descriptor (driver entry point fetched once).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, uint32_t rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

int device_sm_count();

// Host: run `setup` once per (key, current device) and cache its value; the
// first call on a device pays, later calls (from any thread) read the cache.
// A negative result is an error and is not cached.
int once_per_device(const void* key, int (*setup)(const void* key));

// Host: raise a kernel's dynamic shared-memory limit once per device.
cudaError_t set_smem_limit_once(const void* kern, int bytes);

}  // namespace moe
