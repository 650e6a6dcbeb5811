// moe_api.cu — the C ABI (include/moe.h): argument checks, workspace planning,
// TMA descriptor encoding and the launch sequence
//   router -> dispatch -> expert gate/up GEMM -> expert down GEMM (+ combine)
// on the caller's stream, with no host synchronisation. Token tiles combine in
// the down projection's epilogue; the other paths run a combine kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t act_bytes(moe_dtype_t dt) { return dt == MOE_F32 ? 4 : 2; }

// Sizes and dtype only (no pointers).
moe_status_t check_sizes(const moe_args_t* a) {
  if (!a) return MOE_ERR_INVALID_ARG;
  if (a->T < 0 || a->d <= 0 || a->f <= 0) return MOE_ERR_INVALID_ARG;
  if (a->dtype != MOE_F32 && a->dtype != MOE_BF16 && a->dtype != MOE_BF16_INT8W) return MOE_ERR_INVALID_ARG;
  if (a->E != kE || a->k != kK) return MOE_ERR_UNSUPPORTED;
  if (a->T > (int64_t(1) << 24) || a->d > (int64_t(1) << 20) || a->f > (int64_t(1) << 20))
    return MOE_ERR_UNSUPPORTED;
  if (a->dtype == MOE_F32) {
    if (a->d % 64 != 0 || a->f % 64 != 0) return MOE_ERR_UNSUPPORTED;
  } else {
    if (a->d % 256 != 0 || a->f % 128 != 0) return MOE_ERR_UNSUPPORTED;
  }
  // Largest row offset used by the kernels must stay in 32-bit TMA coordinates
  // and the per-expert weight slab in 64-bit addressing.
  if (2 * a->T * std::max(a->d, a->f) > (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_args(const moe_args_t* a) {
  const moe_status_t st = check_sizes(a);
  if (st != MOE_OK || a->T == 0) return st;
  if (!a->x || !a->w_router || !a->w_gate || !a->w_up || !a->w_down || !a->out) return MOE_ERR_INVALID_ARG;
  if (a->dtype == MOE_BF16_INT8W) {
    if (!a->w_scales || !a->w_scales->s_gate || !a->w_scales->s_up || !a->w_scales->s_down)
      return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->w_scales->s_gate) || !aligned16(a->w_scales->s_up) || !aligned16(a->w_scales->s_down))
      return MOE_ERR_MISALIGNED;
  }
  if (!aligned16(a->x) || !aligned16(a->w_router) || !aligned16(a->w_gate) || !aligned16(a->w_up) ||
      !aligned16(a->w_down) || !aligned16(a->out))
    return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

// Signature of cuTensorMapEncodeTiled (driver API), fetched at run time through
// the runtime's entry-point query so the library needs no link-time libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

std::mutex g_cache_mu;
struct DeviceCache {
  void* ws = nullptr;
  size_t bytes = 0;
};
std::vector<DeviceCache> g_cache;

std::vector<int> g_sm_count;
std::mutex g_sm_mu;

}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(g_sm_mu);
  if (static_cast<int>(g_sm_count.size()) <= dev) g_sm_count.resize(dev + 1, 0);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

int once_per_device(const void* key, int (*setup)(const void* key)) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lk(mu);
  const auto k = std::make_pair(key, dev);
  const auto it = cache.find(k);
  if (it != cache.end()) return it->second;
  const int v = setup(key);
  if (v >= 0) cache[k] = v;
  return v;
}

cudaError_t set_smem_limit_once(const void* kern, int bytes) {
  // The kernels' limits are fixed per kernel, so the byte count is looked up
  // through a small registry keyed by the kernel.
  static std::mutex mu;
  static std::map<const void*, int> wanted;
  {
    std::lock_guard<std::mutex> lk(mu);
    wanted[kern] = bytes;
  }
  const int r = once_per_device(kern, [](const void* k) -> int {
    int b = 0;
    {
      std::lock_guard<std::mutex> lk(mu);
      b = wanted[k];
    }
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess ? 1 : -1;
  });
  return r > 0 ? cudaSuccess : cudaErrorInvalidValue;
}

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, uint32_t rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return false;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  for (uint32_t i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (uint32_t i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
  const CUresult r = g_encode(map, dt, rank, const_cast<void*>(base), gdim, gstride, bdim, estride,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool use_weight_stream(int64_t T, moe_path_t path, moe_dtype_t dtype) {
  if (path == MOE_PATH_WEIGHT_STREAM) return true;
  if (path == MOE_PATH_TOKEN_TILE || path == MOE_PATH_TOKEN_TILE_SINGLE) return false;
  // Weight-stream tiles take the tokens on the MMA N side and read each weight
  // byte once; a 128-row token tile of a small batch is mostly padding. Where
  // the crossover lies was measured (interleaved runs at the Grok-1 shape, step
  // ms, weight-stream against 128-row token tiles): int8 weights keep the
  // weight-stream form up to T = 256 (T = 256: 1.76 against 1.97); bf16 weights
  // only up to T = 128 (T = 64: 1.62 against 1.65; T = 160: 1.80 against 1.74;
  // T = 256: 2.11 against 1.67, where the weight-stream down projection's
  // split-K costs most).
  return T <= (dtype == MOE_BF16_INT8W ? 256 : 128);
}

// Expected row tiles of `rows` rows of one expert under balanced routing: a
// token picks the expert with probability 1/4 (two of eight), so its count is
// close to normal with mean m and variance 3m/4; E[ceil(count / rows)] is
// summed over a grid of that density.
double expected_row_tiles(double m, double rows) {
  const double sd = std::sqrt(std::max(0.75 * m, 1e-9));
  double tot = 0.0, wsum = 0.0;
  for (int i = -40; i <= 40; ++i) {
    const double z = i / 10.0, c = m + z * sd, w = std::exp(-0.5 * z * z);
    if (c <= 0.0) continue;
    tot += w * std::ceil(c / rows);
    wsum += w;
  }
  return wsum > 0.0 ? tot / wsum : 0.0;
}

// Split-K factor of the token-tile down projection. Its tiles are long (K = f)
// and few (rows/128 x d/256), so the last partial wave can idle most SMs. Per
// split factor s, estimate the time of the waves of whichever tile form the
// kernels will pick (single-CTA tiles, or CTA-pair 256-row tiles at a 7 %
// discount) from the expected tile counts, plus 20 % of the unsplit work per
// extra split. That cost is fitted to interleaved runs of forced split factors
// (down ms, split 1 / 2 / 4): bf16 T = 160 0.644 / 0.565 / 0.572, T = 384
// 0.677 / 0.608 / 0.632, T = 768 0.843 / 0.935 / 0.935, T = 2048 1.750 / 1.829
// / 1.935; int8 T = 768 1.071 / 0.904 / 0.966, T = 1024 1.025 / 1.152 / 1.329,
// T = 2048 1.965 / 1.972 / 2.118. The model picks the fastest factor at all
// thirteen measured sizes; the earlier one (mean tiles + 0.5 per expert, 2.3 %
// per split for the partial sums' bytes) was up to 16 % off.
int32_t choose_token_tile_down_splits(int64_t T, int64_t d, int64_t f, int32_t requested, bool allow_single,
                                      bool allow_pair, int64_t single_rows) {
  const int64_t kblocks = f / 64;
  if (requested > 0) return kblocks % requested == 0 ? requested : -1;
  auto valid = [&](int64_t s) { return s >= 1 && kblocks % s == 0 && kblocks / s >= 8; };
  const double per_expert = static_cast<double>(2 * T) / kE;
  const double nt = static_cast<double>(d / 256);
  const double t1 = kE * expected_row_tiles(per_expert, static_cast<double>(single_rows)) * nt;  // single-CTA tiles
  const double t2 = kE * expected_row_tiles(per_expert, 256.0) * nt;                                // pair tiles
  const double sms = device_sm_count(), pairs = sms / 2;
  int32_t best = 1;
  double best_t = 1e30;
  for (int64_t s = 1; s <= 8; ++s) {
    if (!valid(s)) continue;
    double t = 1e30;
    if (allow_single) t = std::min(t, std::ceil(t1 * s / sms) / s);
    if (allow_pair) t = std::min(t, std::ceil(t2 * s / pairs) / s / 1.07);
    t += 0.20 * (s - 1) * (t1 / sms);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = static_cast<int32_t>(s);
    }
  }
  return best;
}

int32_t choose_down_splits(int64_t T, int64_t d, int64_t f, int32_t requested) {
  const int64_t kblocks = f / 64;
  auto valid = [&](int64_t s) { return s >= 1 && kblocks % s == 0; };
  if (requested > 0) return valid(requested) ? requested : -1;
  // Enough tiles for ~10 waves over the SMs; keep >= 8 K blocks per split.
  const int64_t base_tiles = ((2 * T) / 128 + kE) * (d / 256);
  int64_t best = 1;
  for (int64_t s = 1; s <= 64; ++s) {
    if (!valid(s) || kblocks / s < 8) continue;
    best = s;
    if (base_tiles * s >= 10 * 148) break;
  }
  return static_cast<int32_t>(best);
}

WorkspaceLayout plan_workspace(int64_t T, int64_t d, int64_t f, moe_dtype_t dtype, moe_path_t path,
                               int32_t down_splits, bool h_external) {
  WorkspaceLayout L{};
  const int64_t rows = 2 * T;
  L.nblk = (T + kRouteTokens - 1) / kRouteTokens;
  L.weight_stream = dtype != MOE_F32 && use_weight_stream(T, path, dtype);
  // Small bf16 batches on the automatic path: the gate/up GEMM in 128-row
  // token tiles (interleaved runs at the Grok-1 shape, gate/up ms against
  // weight-stream tiles: T = 16 0.880 / 0.897, T = 64 1.001-1.014 /
  // 1.047-1.050, T = 128 1.012-1.030 / 1.053-1.057), the down projection in
  // weight-stream tiles (T = 64 0.516-0.531 against 0.585-0.605 ms in token tiles).
  L.gateup_tt = L.weight_stream && path == MOE_PATH_AUTO && dtype == MOE_BF16;
  L.tile_path = dtype != MOE_F32 && (!L.weight_stream || L.gateup_tt);
  if (dtype == MOE_F32) {
    L.splits = 1;
  } else if (L.weight_stream) {
    L.splits = choose_down_splits(T, d, f, down_splits);
  } else {
    // Which token-tile forms may run (see the launch logic in run_forward).
    const bool allow_pair = path == MOE_PATH_TOKEN_TILE || (path == MOE_PATH_AUTO && dtype != MOE_BF16_INT8W);
    const bool allow_single = path != MOE_PATH_TOKEN_TILE;
    // int8 weights take 256-row single-CTA tiles (two MMAs per converted tile).
    L.splits = choose_token_tile_down_splits(T, d, f, down_splits, allow_single, allow_pair,
                                             dtype == MOE_BF16_INT8W ? 256 : 128);
  }
  // A requested split factor must divide the K blocks whichever path runs.
  if (down_splits > 0 && choose_down_splits(T, d, f, down_splits) < 1) L.splits = -1;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.router_slices = router_slices(T, d, dtype);
  L.status = take(kAlign);
  L.arrivals = take(sizeof(int32_t) * L.nblk);  // right after the status word: one memset clears both
  // Arrival counters of the combine in the down-projection epilogue, cleared
  // by the same memset: one per (token, 256-column tile) for token tiles, one
  // per (token, 256-column tile, epilogue warp) for weight-stream tiles.
  L.combine_count = dtype == MOE_F32 ? o : take(sizeof(int32_t) * T * (d / 256) * (L.weight_stream ? 4 : 1));
  L.idx = take(sizeof(int32_t) * rows);
  L.gates = take(sizeof(float) * rows);
  L.hist = take(sizeof(int32_t) * L.nblk * kE);
  L.hist_pre = take(sizeof(int32_t) * (L.nblk + 1) * kE);  // block prefixes + totals (many blocks)
  L.logits_part = L.router_slices > 1 ? take(sizeof(float) * L.router_slices * T * kE) : 0;
  L.counts = take(sizeof(int32_t) * kE);
  L.offsets = take(sizeof(int32_t) * (kE + 1));
  L.perm_token = take(sizeof(int32_t) * rows);
  L.perm_slot = take(sizeof(int32_t) * rows);
  L.slot_pos = take(sizeof(int32_t) * rows);
  L.gate_perm = take(sizeof(float) * rows);
  L.xp = take(act_bytes(dtype) * rows * d);
  L.h = h_external ? 0 : take(act_bytes(dtype) * rows * f);
  L.y = take(sizeof(float) * static_cast<size_t>(std::max(L.splits, 1)) * rows * d);
  L.total = o;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

moe_status_t run_forward(const moe_args_t* a, const moe_options_t* o, const moe_debug_t* dbg, void* workspace,
                         size_t ws_bytes, cudaStream_t stream) {
  const moe_options_t defaults{};
  if (!o) o = &defaults;
  if (o->activation < MOE_ACT_GELU_TANH || o->activation > MOE_ACT_SILU) return MOE_ERR_INVALID_ARG;
  if (o->renormalize != 0 && o->renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (o->post_norm_weight && !(o->norm_eps > 0.0f)) return MOE_ERR_INVALID_ARG;
  if ((o->post_norm_weight && !aligned16(o->post_norm_weight)) || (o->residual && !aligned16(o->residual)))
    return MOE_ERR_MISALIGNED;
  if (o->path < MOE_PATH_AUTO || o->path > MOE_PATH_TOKEN_TILE_SINGLE) return MOE_ERR_INVALID_ARG;
  if (o->down_splits < 0) return MOE_ERR_INVALID_ARG;
  if (o->row_gather != 0 && o->row_gather != 1) return MOE_ERR_INVALID_ARG;
  if (o->separate_combine != 0 && o->separate_combine != 1) return MOE_ERR_INVALID_ARG;
  // The int8-weight GEMMs take fp16 activations from the dispatch copy; a row
  // gather would feed them x's bf16 rows.
  if (o->row_gather == 1 && a->dtype == MOE_BF16_INT8W) return MOE_ERR_UNSUPPORTED;
  if (o->router_bias && !aligned16(o->router_bias)) return MOE_ERR_MISALIGNED;
  const bool h_ext = dbg && dbg->h;
  if (h_ext && !aligned16(dbg->h)) return MOE_ERR_MISALIGNED;
  const WorkspaceLayout L = plan_workspace(a->T, a->d, a->f, a->dtype, o->path, o->down_splits, h_ext);
  if (L.splits < 1) return MOE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < L.total)
    return MOE_ERR_WORKSPACE;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  // Tile counters of the token-tile GEMM launches (pair gate/up, pair down,
  // single-CTA gate/up, single-CTA down), in the status slot (zeroed with it
  // below).
  int32_t* tile_counters = reinterpret_cast<int32_t*>(ws + L.status + 16);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* gates = reinterpret_cast<float*>(ws + L.gates);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* hist_pre = reinterpret_cast<int32_t*>(ws + L.hist_pre);
  int32_t* arrivals = reinterpret_cast<int32_t*>(ws + L.arrivals);
  float* logits_part = L.router_slices > 1 ? reinterpret_cast<float*>(ws + L.logits_part) : nullptr;
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_token = reinterpret_cast<int32_t*>(ws + L.perm_token);
  int32_t* perm_slot = reinterpret_cast<int32_t*>(ws + L.perm_slot);
  int32_t* slot_pos = reinterpret_cast<int32_t*>(ws + L.slot_pos);
  float* gate_perm = reinterpret_cast<float*>(ws + L.gate_perm);
  // With the row gather the token-tile GEMM reads x itself and the dispatch
  // stage skips the permuted copy.
  const bool gather_x = L.tile_path && o->row_gather == 1;
  void* xp = gather_x ? nullptr : static_cast<void*>(ws + L.xp);
  void* h = h_ext ? dbg->h : static_cast<void*>(ws + L.h);
  float* y = reinterpret_cast<float*>(ws + L.y);
  const int64_t T = a->T, d = a->d, f = a->f;
  // The down projection's epilogue sums each token's rows (token tiles and
  // weight-stream tiles); a separate combine kernel runs for the fp32 path,
  // with the post-RMSNorm (it needs whole rows), or when asked for.
  const bool fused_combine = a->dtype != MOE_F32 && !o->post_norm_weight && o->separate_combine == 0;
  int32_t* combine_count = reinterpret_cast<int32_t*>(ws + L.combine_count);

#define MOE_TRY(call)                                  \
  do {                                                 \
    if ((call) != cudaSuccess) return MOE_ERR_CUDA;    \
  } while (0)

  auto mark = [&](int i) {
    return o->stage_events ? cudaEventRecord(static_cast<cudaEvent_t>(o->stage_events[i]), stream) : cudaSuccess;
  };
  // Status word, router arrival counters and combine arrival counters start at
  // zero (contiguous regions, up to the next one).
  MOE_TRY(cudaMemsetAsync(status, 0, L.idx - L.status, stream));
  MOE_TRY(mark(0));
  if (small_route_dispatch(T, d, xp)) {
    // Decode-sized batches: router and dispatch in one cluster launch.
    MOE_TRY(launch_route_dispatch_small(a->dtype, a->x, a->w_router, o->router_bias, T, d, o->renormalize, idx,
                                        gates, counts, offsets, perm_token, perm_slot, slot_pos, gate_perm, xp,
                                        status, stream));
    MOE_TRY(mark(1));
  } else {
    MOE_TRY(launch_router(a->dtype, a->x, a->w_router, o->router_bias, T, d, o->renormalize, L.router_slices,
                          logits_part, arrivals, idx, gates, hist, stream));
    MOE_TRY(mark(1));
    MOE_TRY(launch_dispatch(a->dtype, a->x, T, d, L.nblk, idx, gates, hist, hist_pre, counts, offsets,
                            perm_token, perm_slot, slot_pos, gate_perm, xp, status, stream));
  }
  MOE_TRY(mark(2));
  if (a->dtype == MOE_F32) {
    MOE_TRY(launch_f32_gateup(static_cast<const float*>(xp), static_cast<const float*>(a->w_gate),
                              static_cast<const float*>(a->w_up), counts, offsets, T, d, f, o->activation,
                              static_cast<float*>(h), status, stream));
    MOE_TRY(mark(3));
    MOE_TRY(launch_f32_down(static_cast<const float*>(h), static_cast<const float*>(a->w_down), counts, offsets,
                            gate_perm, T, d, f, y, status, stream));
  } else {
    const bool w8 = a->dtype == MOE_BF16_INT8W;
    TcGemmArgs g{};
    g.x = gather_x ? a->x : xp;
    g.row_token = gather_x ? perm_token : nullptr;
    g.x_rows = T;
    g.w0 = a->w_gate;
    g.w1 = a->w_up;
    g.s0 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_gate) : nullptr;
    g.s1 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_up) : nullptr;
    g.counts = counts;
    g.offsets = offsets;
    g.gate_perm = gate_perm;
    g.out = h;
    g.rows = 2 * T;
    g.K = static_cast<int32_t>(d);
    g.N = static_cast<int32_t>(f);
    g.splits = 1;
    g.act = o->activation;
    g.int8_weights = w8;
    g.weight_stream = L.weight_stream && !L.gateup_tt;
    // Small batches (<= 32 token slots per expert on average): weight-stream
    // tiles of at most 64 tokens, which leave room for more weight stages in flight.
    g.short_tiles = g.weight_stream && T <= 128;
    g.status = status;
    g.tile_counter = tile_counters;
    g.tile_counter_single = tile_counters + 2;
    // Token tiles: with MOE_PATH_AUTO both forms are launched and the kernels
    // pick one of them on the device from the expert counts (the other returns
    // at once); TOKEN_TILE / TOKEN_TILE_SINGLE force one form.
    // int8 weights always take single CTAs under AUTO: their pair form waits on
    // both CTAs' converters every stage and measured slower.
    const bool auto_tt = !L.weight_stream && o->path == MOE_PATH_AUTO && !w8;
    const bool run_pair = !L.weight_stream && o->path != MOE_PATH_TOKEN_TILE_SINGLE &&
                          !(w8 && o->path == MOE_PATH_AUTO);
    const bool run_single = L.weight_stream || o->path != MOE_PATH_TOKEN_TILE;
    auto launch_gemm = [&](TcGemmArgs args, bool down) -> cudaError_t {
      if (run_pair) {
        args.select = auto_tt ? 1 : 0;
        const cudaError_t e = down ? launch_tc_down_pair(args, stream) : launch_tc_gateup_pair(args, stream);
        if (e != cudaSuccess) return e;
      }
      if (run_single) {
        args.select = auto_tt ? 2 : 0;
        return down ? launch_tc_down(args, stream) : launch_tc_gateup(args, stream);
      }
      return cudaSuccess;
    };
    // bf16 gate/up under AUTO with at least kTallMinT tokens (128 rows per
    // expert on average): 256-row tiles on single CTAs, which beat both
    // 128-row forms there (measured gate/up with sixteen epilogue warps, two
    // runs: T = 384 1.11 against 1.03 ms, so not below; T = 512 1.20 against
    // 1.21; T = 768 1.31 against 1.34-1.36; T = 4096 5.15-5.39 against
    // 5.67-5.80 before). The down projection keeps the choice above: its
    // epilogue, which 256-row tiles cannot overlap with the next tile, is heavier.
    if (L.gateup_tt) {
      // 128-row token tiles on single CTAs alone: with at most 32 rows per
      // expert on average the CTA-pair form never pays.
      TcGemmArgs gt = g;
      gt.select = 0;
      MOE_TRY(launch_tc_gateup(gt, stream));
    } else if (auto_tt && !gather_x && T >= kTallMinT) {
      TcGemmArgs gt = g;
      gt.tall_tiles = true;
      gt.select = 0;
      MOE_TRY(launch_tc_gateup(gt, stream));
    } else {
      MOE_TRY(launch_gemm(g, false));
    }
    MOE_TRY(mark(3));
    TcGemmArgs g2 = g;
    g2.weight_stream = L.weight_stream;
    g2.short_tiles = L.weight_stream && T <= 128;
    g2.x = h;
    g2.row_token = nullptr;
    g2.w0 = a->w_down;
    g2.w1 = nullptr;
    g2.s0 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_down) : nullptr;
    g2.s1 = nullptr;
    g2.out = y;
    g2.K = static_cast<int32_t>(f);
    g2.N = static_cast<int32_t>(d);
    g2.splits = L.splits;
    g2.tile_counter = tile_counters + 1;
    g2.tile_counter_single = tile_counters + 3;
    if (fused_combine) {
      g2.perm_token = perm_token;
      g2.slot_pos = slot_pos;
      g2.combine_count = combine_count;
      g2.combine_out = a->out;
      g2.residual = o->residual;
    }
    MOE_TRY(launch_gemm(g2, true));
  }
  MOE_TRY(mark(4));
  if (!fused_combine)
    MOE_TRY(launch_combine(a->dtype, y, 2 * T * d, L.splits, slot_pos, T, d, o->residual, o->post_norm_weight,
                           o->norm_eps, a->out, status, stream));
  MOE_TRY(mark(5));

  if (dbg) {
    auto cp = [&](void* dst, const void* src, size_t bytes) {
      return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, stream) : cudaSuccess;
    };
    MOE_TRY(cp(dbg->idx, idx, sizeof(int32_t) * 2 * T));
    MOE_TRY(cp(dbg->gates, gates, sizeof(float) * 2 * T));
    MOE_TRY(cp(dbg->counts, counts, sizeof(int32_t) * kE));
    MOE_TRY(cp(dbg->offsets, offsets, sizeof(int32_t) * (kE + 1)));
    MOE_TRY(cp(dbg->perm_token, perm_token, sizeof(int32_t) * 2 * T));
    MOE_TRY(cp(dbg->perm_slot, perm_slot, sizeof(int32_t) * 2 * T));
  }
#undef MOE_TRY
  return MOE_OK;
}

// Device address of the moe_forward_noalloc scratch's status word on device
// `dev`, or nullptr while no noalloc call has set it up there.
const void* noalloc_status_word(int dev);

}  // namespace

extern "C" {

moe_status_t moe_forward_ex(const moe_args_t* args, const moe_options_t* opts, const moe_debug_t* dbg,
                            void* workspace, size_t ws_bytes, moe_stream_t stream) {
  const moe_status_t st = check_args(args);
  if (st != MOE_OK || args->T == 0) return st;
  return run_forward(args, opts, dbg, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t moe_workspace_size_ex(int64_t T, int64_t d, int64_t f, int32_t E, int32_t k, moe_dtype_t dtype,
                             moe_path_t path, int32_t down_splits) {
  moe_args_t a{};
  a.T = T;
  a.d = d;
  a.f = f;
  a.E = E;
  a.k = k;
  a.dtype = dtype;
  if (T <= 0 || check_sizes(&a) != MOE_OK) return 0;
  if (path < MOE_PATH_AUTO || path > MOE_PATH_TOKEN_TILE_SINGLE) return 0;
  if (down_splits < 0) return 0;
  const WorkspaceLayout L = plan_workspace(T, d, f, dtype, path, down_splits, false);
  if (L.splits < 1) return 0;
  return L.total;
}

size_t moe_workspace_size(int64_t T, int64_t d, int64_t f, int32_t E, int32_t k, moe_dtype_t dtype) {
  return moe_workspace_size_ex(T, d, f, E, k, dtype, MOE_PATH_AUTO, 0);
}

moe_status_t moe_forward(const void* x, const float* w_router, const void* w_gate, const void* w_up,
                         const void* w_down, const moe_scales_t* w_scales, void* out, int64_t T, int64_t d,
                         int64_t f, int32_t E, int32_t k, moe_dtype_t dtype, moe_stream_t stream) {
  moe_args_t a{x, w_router, w_gate, w_up, w_down, w_scales, out, T, d, f, E, k, dtype};
  const moe_status_t st = check_args(&a);
  if (st != MOE_OK || T == 0) return st;
  const size_t need = moe_workspace_size(T, d, f, E, k, dtype);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_cache_mu);
  if (static_cast<int>(g_cache.size()) <= dev) g_cache.resize(dev + 1);
  DeviceCache& c = g_cache[dev];
  if (c.bytes < need) {
    // The previous buffer may still be in use by queued work on any stream.
    if (c.ws) {
      if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
      cudaFree(c.ws);
      c.ws = nullptr;
      c.bytes = 0;
    }
    if (cudaMalloc(&c.ws, need) != cudaSuccess) {
      c.ws = nullptr;
      return MOE_ERR_CUDA;
    }
    c.bytes = need;
  }
  return run_forward(&a, nullptr, nullptr, c.ws, c.bytes, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_device_status(const void* workspace, moe_stream_t stream, uint32_t* code) {
  // The status words to read: the given workspace's, or with NULL both
  // library-owned ones of the current device (the moe_forward cache and the
  // moe_forward_noalloc scratch), whichever exist.
  const void* words[2] = {workspace, nullptr};
  if (!workspace) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    {
      std::lock_guard<std::mutex> lk(g_cache_mu);
      words[0] = static_cast<int>(g_cache.size()) > dev ? g_cache[dev].ws : nullptr;
    }
    words[1] = noalloc_status_word(dev);
  }
  uint32_t v[2] = {0, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < 2; ++i)
    if (words[i] && cudaMemcpyAsync(&v[i], words[i], sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  const uint32_t all = v[0] | v[1];
  if (code) *code = all;
  return all == 0 ? MOE_OK : MOE_ERR_DEVICE_CHECK;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size or configuration";
    case MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed (see moe_device_status code)";
  }
  return "unknown status";
}

int32_t moe_abi_version(void) { return 2; }

int32_t moe_build_flags(void) { return kDebugBounds ? MOE_BUILD_DEBUG_BOUNDS : 0; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Expert-parallel building blocks (Grok-1 book ch. 1, section 1.6.3: the MoE
// layer shards the expert axis over the devices of the mesh). A forward over
// W GPUs routes and dispatches each GPU's own tokens (moe_route_dispatch),
// sends each block of rows to the GPU that owns its experts, runs the local
// experts on the rows it received (moe_experts_forward, after moe_gather_rows
// has made them expert-contiguous), sends the gate-scaled rows back and sums
// each token's two rows (moe_combine). The exchanges themselves belong to the
// caller's communication library.
// ---------------------------------------------------------------------------

namespace {

struct RouteLayout {
  size_t status, arrivals, logits_part, hist, hist_pre, total;
  int64_t nblk;
  int32_t slices;
};

RouteLayout plan_route(int64_t T, int64_t d, moe_dtype_t dtype) {
  RouteLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.nblk = (T + kRouteTokens - 1) / kRouteTokens;
  L.slices = router_slices(T, d, dtype);
  L.status = take(kAlign);
  L.arrivals = take(sizeof(int32_t) * L.nblk);
  L.logits_part = L.slices > 1 ? take(sizeof(float) * L.slices * T * kE) : 0;
  L.hist = take(sizeof(int32_t) * L.nblk * kE);
  L.hist_pre = take(sizeof(int32_t) * (L.nblk + 1) * kE);
  L.total = o;
  return L;
}

struct ExpertsLayout {
  size_t status, counts, offsets, ones, h, ypart, total;
  int32_t splits;
  bool weight_stream;  // down projection (and gate/up unless gateup_tt) in weight-stream tiles
  bool gateup_tt;      // bf16, automatic path: gate/up in 128-row token tiles (as in the whole layer)
};

bool experts_sizes_ok(int64_t R, int64_t d, int64_t f, int32_t n, moe_dtype_t dtype) {
  moe_args_t a{};
  a.T = (R + 1) / 2;
  a.d = d;
  a.f = f;
  a.E = kE;
  a.k = kK;
  a.dtype = dtype;
  return R >= 0 && R <= (int64_t(1) << 25) && n >= 1 && n <= kE && check_sizes(&a) == MOE_OK;
}

ExpertsLayout plan_experts(int64_t R, int64_t d, int64_t f, int32_t n, moe_dtype_t dtype, moe_path_t path,
                           int32_t down_splits) {
  ExpertsLayout L{};
  // Weight-stream tiles when the local experts hold few rows on average (as in
  // the whole-layer choice: <= 64 with int8 weights, <= 32 with bf16), token
  // tiles otherwise.
  const int64_t ws_rows = dtype == MOE_BF16_INT8W ? 64 : 32;
  L.weight_stream = dtype != MOE_F32 && (path == MOE_PATH_WEIGHT_STREAM ||
                                         (path == MOE_PATH_AUTO && R <= ws_rows * static_cast<int64_t>(n)));
  L.gateup_tt = L.weight_stream && path == MOE_PATH_AUTO && dtype == MOE_BF16;
  const int64_t kblocks = f / 64;
  if (down_splits > 0) {
    L.splits = kblocks % down_splits == 0 && dtype != MOE_F32 ? down_splits : (down_splits == 1 ? 1 : -1);
  } else if (L.weight_stream) {
    // Enough tiles for ~10 waves, at least 8 K blocks per split.
    const int64_t base = (R / 128 + n) * (d / 256);
    int64_t best = 1;
    for (int64_t s = 1; s <= 64; ++s) {
      if (kblocks % s != 0 || kblocks / s < 8) continue;
      best = s;
      if (base * s >= 10 * static_cast<int64_t>(device_sm_count())) break;
    }
    L.splits = static_cast<int32_t>(best);
  } else {
    L.splits = 1;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.status = take(kAlign);
  L.counts = take(sizeof(int32_t) * kE);
  L.offsets = take(sizeof(int32_t) * (kE + 1));
  L.ones = take(sizeof(float) * std::max<int64_t>(R, 1));
  L.h = take(act_bytes(dtype) * std::max<int64_t>(R, 1) * f);
  L.ypart = L.splits > 1 ? take(sizeof(float) * L.splits * R * d) : o;
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

size_t moe_route_workspace_size(int64_t T, int64_t d, moe_dtype_t dtype) {
  moe_args_t a{};
  a.T = T;
  a.d = d;
  a.f = 128;
  a.E = kE;
  a.k = kK;
  a.dtype = dtype;
  if (T <= 0 || check_sizes(&a) != MOE_OK) return 0;
  return plan_route(T, d, dtype).total;
}

moe_status_t moe_route_dispatch(const void* x, const float* w_router, const float* router_bias, int64_t T,
                                int64_t d, moe_dtype_t dtype, int32_t renormalize, const moe_routed_t* r,
                                void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_args_t a{};
  a.T = T;
  a.d = d;
  a.f = 128;
  a.E = kE;
  a.k = kK;
  a.dtype = dtype;
  moe_status_t st = check_sizes(&a);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !r || !r->idx || !r->gates || !r->counts || !r->offsets || !r->perm_token ||
      !r->perm_slot || !r->slot_pos || !r->gate_perm || !r->xp)
    return MOE_ERR_INVALID_ARG;
  if (renormalize != 0 && renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(r->xp) || (router_bias && !aligned16(router_bias)))
    return MOE_ERR_MISALIGNED;
  const RouteLayout L = plan_route(T, d, dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < L.total)
    return MOE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  if (cudaMemsetAsync(status, 0, L.logits_part ? L.logits_part - L.status : L.hist - L.status, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (small_route_dispatch(T, d, r->xp))
    return launch_route_dispatch_small(dtype, x, w_router, router_bias, T, d, renormalize, r->idx, r->gates,
                                       r->counts, r->offsets, r->perm_token, r->perm_slot, r->slot_pos,
                                       r->gate_perm, r->xp, status, s) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  if (launch_router(dtype, x, w_router, router_bias, T, d, renormalize, L.slices,
                    L.slices > 1 ? reinterpret_cast<float*>(ws + L.logits_part) : nullptr,
                    reinterpret_cast<int32_t*>(ws + L.arrivals), r->idx, r->gates, hist, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_dispatch(dtype, x, T, d, L.nblk, r->idx, r->gates, hist, reinterpret_cast<int32_t*>(ws + L.hist_pre),
                      r->counts, r->offsets, r->perm_token, r->perm_slot, r->slot_pos, r->gate_perm, r->xp, status,
                      s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

size_t moe_experts_workspace_size(int64_t R, int64_t d, int64_t f, int32_t n_experts, moe_dtype_t dtype,
                                  moe_path_t path, int32_t down_splits) {
  if (R <= 0 || !experts_sizes_ok(R, d, f, n_experts, dtype)) return 0;
  if (path < MOE_PATH_AUTO || path > MOE_PATH_TOKEN_TILE_SINGLE || down_splits < 0) return 0;
  const ExpertsLayout L = plan_experts(R, d, f, n_experts, dtype, path, down_splits);
  return L.splits < 1 ? 0 : L.total;
}

moe_status_t moe_experts_forward(const moe_expert_rows_t* a, const moe_options_t* opts, void* workspace,
                                 size_t ws_bytes, moe_stream_t stream) {
  if (!a) return MOE_ERR_INVALID_ARG;
  const moe_options_t defaults{};
  const moe_options_t* o = opts ? opts : &defaults;
  if (a->dtype != MOE_F32 && a->dtype != MOE_BF16 && a->dtype != MOE_BF16_INT8W) return MOE_ERR_INVALID_ARG;
  if (a->R < 0 || a->d <= 0 || a->f <= 0 || a->n_experts < 1 || a->n_experts > kE) return MOE_ERR_INVALID_ARG;
  if (!experts_sizes_ok(a->R, a->d, a->f, a->n_experts, a->dtype)) return MOE_ERR_UNSUPPORTED;
  if (a->R == 0) return MOE_OK;
  if (o->activation < MOE_ACT_GELU_TANH || o->activation > MOE_ACT_SILU) return MOE_ERR_INVALID_ARG;
  if (o->path < MOE_PATH_AUTO || o->path > MOE_PATH_TOKEN_TILE_SINGLE || o->down_splits < 0)
    return MOE_ERR_INVALID_ARG;
  if (!a->xp || !a->counts || !a->w_gate || !a->w_up || !a->w_down || !a->y) return MOE_ERR_INVALID_ARG;
  const bool w8 = a->dtype == MOE_BF16_INT8W;
  if (w8 && (!a->w_scales || !a->w_scales->s_gate || !a->w_scales->s_up || !a->w_scales->s_down))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(a->xp) || !aligned16(a->w_gate) || !aligned16(a->w_up) || !aligned16(a->w_down) ||
      !aligned16(a->y))
    return MOE_ERR_MISALIGNED;
  if (w8 && (!aligned16(a->w_scales->s_gate) || !aligned16(a->w_scales->s_up) || !aligned16(a->w_scales->s_down)))
    return MOE_ERR_MISALIGNED;
  const ExpertsLayout L = plan_experts(a->R, a->d, a->f, a->n_experts, a->dtype, o->path, o->down_splits);
  if (L.splits < 1) return MOE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < L.total)
    return MOE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  float* ones = reinterpret_cast<float*>(ws + L.ones);
  void* h = ws + L.h;
  const int64_t R = a->R, d = a->d, f = a->f;
  const float* gate = a->gate ? a->gate : ones;
  if (cudaMemsetAsync(status, 0, kAlign, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_local_schedule(a->counts, a->n_experts, counts, offsets, a->gate ? nullptr : ones, R, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // The row-count-based launch sizes of the kernels take T = R / 2 (R rows).
  const int64_t T_eq = (R + 1) / 2;
  if (a->dtype == MOE_F32) {
    if (launch_f32_gateup(static_cast<const float*>(a->xp), static_cast<const float*>(a->w_gate),
                          static_cast<const float*>(a->w_up), counts, offsets, T_eq, d, f, o->activation,
                          static_cast<float*>(h), status, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (launch_f32_down(static_cast<const float*>(h), static_cast<const float*>(a->w_down), counts, offsets, gate,
                        T_eq, d, f, a->y, status, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  float* y = L.splits > 1 ? reinterpret_cast<float*>(ws + L.ypart) : a->y;
  TcGemmArgs g{};
  g.x = a->xp;
  g.x_rows = R;
  g.w0 = a->w_gate;
  g.w1 = a->w_up;
  g.s0 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_gate) : nullptr;
  g.s1 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_up) : nullptr;
  g.counts = counts;
  g.offsets = offsets;
  g.gate_perm = gate;
  g.out = h;
  g.rows = R;
  g.K = static_cast<int32_t>(d);
  g.N = static_cast<int32_t>(f);
  g.splits = 1;
  g.act = o->activation;
  g.int8_weights = w8;
  g.weight_stream = L.weight_stream && !L.gateup_tt;
  g.short_tiles = g.weight_stream && R <= 32 * static_cast<int64_t>(a->n_experts);
  g.status = status;
  g.n_experts = a->n_experts;
  // One token-tile form per call here (the single-CTA one unless the pair form
  // is asked for): the device-side choice between them needs zeroed tile
  // counters that this workspace does not keep.
  const bool pair = !L.weight_stream && o->path == MOE_PATH_TOKEN_TILE;
  auto gemm = [&](const TcGemmArgs& args, bool down) -> cudaError_t {
    if (pair) return down ? launch_tc_down_pair(args, s) : launch_tc_gateup_pair(args, s);
    return down ? launch_tc_down(args, s) : launch_tc_gateup(args, s);
  };
  if (gemm(g, false) != cudaSuccess) return MOE_ERR_CUDA;
  TcGemmArgs g2 = g;
  g2.weight_stream = L.weight_stream;
  g2.short_tiles = L.weight_stream && R <= 32 * static_cast<int64_t>(a->n_experts);
  g2.x = h;
  g2.w0 = a->w_down;
  g2.w1 = nullptr;
  g2.s0 = w8 ? static_cast<const __nv_bfloat16*>(a->w_scales->s_down) : nullptr;
  g2.s1 = nullptr;
  g2.out = y;
  g2.K = static_cast<int32_t>(f);
  g2.N = static_cast<int32_t>(d);
  g2.splits = L.splits;
  if (gemm(g2, true) != cudaSuccess) return MOE_ERR_CUDA;
  if (L.splits > 1 && launch_sum_splits(y, R * d, L.splits, R * d, a->y, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_combine(const float* y, const int32_t* slot_pos, int64_t T, int64_t d, moe_dtype_t dtype,
                         const void* residual, const float* post_norm_weight, float norm_eps, void* out,
                         void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || d <= 0 || d % 4 != 0 || T > (int64_t(1) << 24)) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_F32 && dtype != MOE_BF16 && dtype != MOE_BF16_INT8W) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !slot_pos || !out) return MOE_ERR_INVALID_ARG;
  if (post_norm_weight && !(norm_eps > 0.0f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out) || (residual && !aligned16(residual)) ||
      (post_norm_weight && !aligned16(post_norm_weight)))
    return MOE_ERR_MISALIGNED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < kAlign)
    return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, kAlign, s) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_combine(dtype, y, 2 * T * d, 1, slot_pos, T, d, residual, post_norm_weight, norm_eps, out, status,
                        s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int32_t* index, int64_t n,
                             int64_t row_bytes, void* dst, void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (n < 0 || src_rows < 0 || row_bytes <= 0 || row_bytes % 4 != 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!src || !index || !dst) return MOE_ERR_INVALID_ARG;
  const uintptr_t a = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst);
  if ((a & (row_bytes % 16 == 0 ? 15u : 3u)) != 0) return MOE_ERR_MISALIGNED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < kAlign)
    return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, kAlign, s) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_gather_rows(src, src_rows, index, n, row_bytes, dst, status, s) == cudaSuccess ? MOE_OK
                                                                                             : MOE_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_forward_noalloc: the forward pass with its scratch in a fixed,
// library-owned device array instead of memory the caller or the library
// allocates at call time.
//
// Who needs it: code that must not call cudaMalloc while it runs, for example a
// host framework that reserves all device memory in its own pool at start-up
// (an allocation behind its back could fail late or break its accounting), or
// a latency-critical loop where cudaMalloc / cudaFree would stall on a device
// synchronisation. Such callers pass inputs and outputs only.
//
// The scratch is a static __device__ array of kNoAllocScratchBytes per device;
// every GPU that loads this library holds it until the process exits. Host
// code must not use the array's name as a device address (on the host it is
// only a stand-in symbol), so the device address is fetched once per device
// with cudaGetSymbolAddress while that device is current, on the first call
// made on that device. That first call should therefore happen before any
// stream capture. All calls on a device share the one array and leave their
// contents in it: calls whose work may overlap on the GPU (different streams
// without ordering) race on it. Each call clears the status word it uses; the
// other scratch regions are fully written before they are read.
// ---------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
std::vector<void*> g_noalloc_ptr;  // per device: device address of g_noalloc_scratch

const void* noalloc_status_word(int dev) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  // run_forward keeps the status word at offset 0 of the scratch.
  return static_cast<int>(g_noalloc_ptr.size()) > dev ? g_noalloc_ptr[dev] : nullptr;
}

// Device address of the scratch array on the current device (set up once).
cudaError_t noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (static_cast<int>(g_noalloc_ptr.size()) <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_forward_noalloc(const moe_args_t* args, const moe_options_t* opts,
                                            moe_stream_t stream) {
  const moe_status_t st = check_args(args);
  if (st != MOE_OK) return st;
  // Look the scratch up first, so that a T == 0 call (which launches nothing)
  // serves as the device's set-up call before any stream capture.
  void* ws = nullptr;
  if (noalloc_scratch_address(&ws) != cudaSuccess) return MOE_ERR_CUDA;
  if (args->T == 0) return MOE_OK;
  moe_options_t o{};
  if (opts) o = *opts;
  if (o.down_splits < 0) return MOE_ERR_INVALID_ARG;
  WorkspaceLayout L = plan_workspace(args->T, args->d, args->f, args->dtype, o.path, o.down_splits, false);
  if (L.splits < 1) return MOE_ERR_UNSUPPORTED;
  if (L.total > kNoAllocScratchBytes && o.down_splits == 0 && L.splits > 1) {
    // Automatic split-K: take the largest factor below the automatic one whose
    // partial sums still fit the fixed scratch.
    for (int32_t s = L.splits - 1; s >= 1; --s) {
      const WorkspaceLayout C = plan_workspace(args->T, args->d, args->f, args->dtype, o.path, s, false);
      if (C.splits == s && C.total <= kNoAllocScratchBytes) {
        o.down_splits = s;
        L = C;
        break;
      }
    }
  }
  if (L.total > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;  // problem too large for the fixed scratch
  return run_forward(args, &o, nullptr, ws, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}
