// gemm_common.cuh — pieces shared by the single-CTA and the CTA-pair grouped
// expert GEMM kernels: tile constants, parameters, the device-side tile
// scheduler data, the gate activation, the exact int8 -> fp16 conversion and the token-tile
// epilogue (act(gate) * up -> bf16 H, or gate * down -> fp32 Y).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "moe_internal.cuh"
#include "sm100.cuh"
#include "tile_order.cuh"

namespace moe {
namespace tc {

using namespace moe::sm100;

constexpr int BM = 128;                 // tile rows (tokens) per CTA
constexpr int BK = 64;                  // K per stage: 64 bf16 = one 128-B swizzle row
constexpr int X_BYTES = BM * BK * 2;    // 16 KB
constexpr int WCHUNK = BK * 64 * 2;     // 8 KB: [64 K x 64 N] bf16, 128-B swizzle
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: no wait is unbounded
constexpr long long kL2GroupBytes = 64ll << 20;     // activation rows of one row-tile group
constexpr long long kL2UngroupedBytes = 96ll << 20; // an expert's rows above this are grouped

enum { GATEUP = 0, DOWN = 1 };

struct Params {
  const int32_t* counts;
  const int32_t* offsets;
  const float* gate_perm;
  const int32_t* row_token;  // GATEUP token tiles: token of each permuted row, A rows gathered from x
  const __nv_bfloat16* s0;
  const __nv_bfloat16* s1;
  void* out;
  int64_t rows;          // total permuted rows (2T)
  int64_t split_stride;  // elements between split-K partial buffers (DOWN)
  int32_t K, N;
  int32_t splits;
  int32_t kb_per_split;  // 64-deep K blocks per tile
  int32_t ntile;         // output columns per tile (128 GATEUP, 256 DOWN)
  int32_t act;           // moe_activation_t of the gate branch
  int32_t select;        // kRunAlways, or run only if the pair / single form is preferred
  int32_t sm_count;      // SMs of the device (same value for both token-tile kernels)
  int32_t* tile_counter; // tiles handed out in order (zero on entry), or nullptr (static order)
  int32_t group_rows;    // row tiles per L2 group (tile_order.cuh) ...
  int32_t group_limit;   // ... for experts with more row tiles than this
  uint32_t* status;
  // DOWN token tiles with the combine in the epilogue (combine_count != nullptr)
  const int32_t* perm_token;
  const int32_t* slot_pos;
  int32_t* combine_count;
  __nv_bfloat16* combine_out;
  const __nv_bfloat16* residual;
};

enum { kRunAlways = 0, kRunIfPair = 1, kRunIfSingle = 2 };

// Token tiles can run as 128-row tiles on single CTAs or as 256-row tiles on
// CTA pairs. Which is faster depends on the per-expert counts (only known on
// the device): pair tiles move a third less operand data per MMA but pad each
// expert's row count up to a multiple of 256 instead of 128, and both forms
// lose their last partial wave. Both kernels evaluate this on the same counts
// and agree; the pair form is taken when its waves, discounted by 7 %, are fewer
// (measured: a pair tile, with its tiles handed out in order, runs about 7 %
// faster than two single-CTA tiles of the same rows).
__device__ __forceinline__ bool pair_preferred(const Params& p) {
  int64_t single_tiles = 0, pair_tiles = 0;
  for (int e = 0; e < kE; ++e) {
    const int c = p.counts[e];
    single_tiles += (c + 127) / 128;
    pair_tiles += (c + 255) / 256;
  }
  const int64_t per = static_cast<int64_t>(p.N / p.ntile) * p.splits;
  const int64_t sms = p.sm_count, pairs = p.sm_count / 2;
  const int64_t w_single = (single_tiles * per + sms - 1) / sms;
  const int64_t w_pair = (pair_tiles * per + pairs - 1) / pairs;
  return w_pair * 100 < w_single * 107;
}

// True if this launch should do nothing (the other token-tile form runs).
__device__ __forceinline__ bool skip_launch(const Params& p) {
  if (p.select == kRunAlways) return false;
  return pair_preferred(p) != (p.select == kRunIfPair);
}

struct SharedSched {
  int32_t cnt[kE];
  int32_t off[kE];
  int32_t mt[kE];
  int32_t pre[kE + 1];
};

struct Tile {
  int e, row0, rows, n0, kb0;
};

// Token ids of one producer lane's four A rows (permuted rows q0 .. q0+3 of a
// tile whose valid rows are [t.row0, t.row0 + t.rows)). Rows past the expert's
// count repeat the tile's first token: they are computed and never stored.
__device__ __forceinline__ void gather_rows(const Params& p, const Tile& t, int q0, int32_t r[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int q = q0 + j;
    r[j] = __ldg(p.row_token + (q < t.row0 + t.rows ? q : t.row0));
  }
}

// Row tiles of `tile_rows` per expert, column tiles of p.ntile, splits; row
// tile fastest so that concurrently running CTAs share weight tiles in L2.
__device__ __forceinline__ void build_sched(SharedSched& s, const Params& p, int tile_rows) {
  int acc = 0;
  const int nt_count = p.N / p.ntile;
  for (int e = 0; e < kE; ++e) {
    const int c = p.counts[e];
    s.cnt[e] = c;
    s.off[e] = p.offsets[e];
    s.mt[e] = (c + tile_rows - 1) / tile_rows;
    s.pre[e] = acc;
    acc += s.mt[e] * nt_count * p.splits;
  }
  s.pre[kE] = acc;
  if (kDebugBounds && !expert_blocks_ok(p.counts, p.offsets, kE, p.rows)) {
    atomicOr(p.status, kStatusBounds);
    s.pre[kE] = 0;  // no tile: every role sees the same empty schedule
  }
}

__device__ __forceinline__ bool decode_tile(const SharedSched& s, const Params& p, int tile, int tile_rows,
                                            Tile& t) {
  if (tile >= s.pre[kE]) return false;
  int e = 0;
  while (tile >= s.pre[e + 1]) ++e;
  int mt, nt, ks;
  tile_coords(tile - s.pre[e], s.mt[e], p.N / p.ntile, group_for(s.mt[e], p.group_rows, p.group_limit), mt, nt, ks);
  t.e = e;
  t.row0 = s.off[e] + mt * tile_rows;
  t.rows = min(tile_rows, s.cnt[e] - mt * tile_rows);
  t.n0 = nt * p.ntile;
  t.kb0 = ks * p.kb_per_split;
  if (kDebugBounds && !tile_ok(t.row0, t.rows, p.rows, t.n0, p.ntile, p.N)) {
    atomicOr(p.status, kStatusBounds);
    return false;  // every role decodes the same tile and stops here
  }
  return true;
}

// Hardware tanh (PTX tanh.approx.f32, relative error ~2^-11): below the bf16
// rounding that H receives right after, and a single instruction, which keeps
// the epilogue from taking issue slots the int8 converters need.
__device__ __forceinline__ float tanh_hw(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Gate-branch activation: GELU (tanh form or erf form) or SiLU, the latter as
// z * sigmoid(z) = 0.5 z (1 + tanh(z / 2)).
__device__ __forceinline__ float act_f32(float z, int mode) {
  if (mode == MOE_ACT_GELU_ERF) return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
  if (mode == MOE_ACT_SILU) return 0.5f * z * (1.0f + tanh_hw(0.5f * z));
  const float u = 0.7978845608028654f * (z + 0.044715f * z * z * z);
  return 0.5f * z * (1.0f + tanh_hw(u));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Nonzero if either fp16 half of `h` is infinite or NaN (exponent all ones).
__device__ __forceinline__ uint32_t f16x2_nonfinite(uint32_t h) {
  return static_cast<uint32_t>((h & 0x7C00u) == 0x7C00u) | static_cast<uint32_t>((h & 0x7C000000u) == 0x7C000000u);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t v;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(v) : "f"(hi), "f"(lo));  // upper half from the first source
  return v;
}

// Four int8 values (one 32-bit word) -> four fp16 (two 32-bit words), exact:
// flip the sign bit to get q + 128 in [0, 255], make it the low mantissa byte of
// fp16 1024 (0x6400: exponent 2^10, unit mantissa step), so each half is
// 1024 + q + 128, then one packed subtraction of 1152 leaves q. Both operands lie
// in [1024, 2048), so the difference is exact, and every |q| <= 128 is an fp16.
__device__ __forceinline__ void i8x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);  // halves 0x64:b0, 0x64:b1
  const uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);  // halves 0x64:b2, 0x64:b3
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0x64806480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0x64806480u));
}

// Convert 16-byte int8 segment `seg` of a staging area made of [64 K][128 N]
// int8 boxes into the fp16 weight tile: box b covers fp16 chunks 2b and 2b+1,
// each [64 K][64 N] with the 128-B swizzle (16-B unit u of row k is stored at
// unit u ^ (k % 8)).
//
// Segment order. 16-byte shared-memory accesses are served eight threads at a
// time, and each group of eight must touch eight different 16-B bank groups to
// take one pass. Within every 16 consecutive segments (one row pair k, k+1) the
// first eight take columns 0-3 of row k and 4-7 of row k+1, the next eight the
// rest: the loads (unswizzled staging, unit = c16) then hit units 0..7, and the
// two swizzled stores of a group land on units (u ^ k) with u = 0, 2, 4, 6 for
// the even row and on the odd units for the odd row, again all eight distinct.
// (Row-major order, eight groups of one row, wrote every unit twice: one per
// 64-column chunk.)
// Bounded wait taken by a whole warp: every lane waits, and the warp goes on
// only if every lane saw the phase complete and no role has aborted, so the
// warp-synchronous instructions after it (tcgen05.ld, __syncwarp) never run on
// part of a warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, kWaitLimitNs) && !*abort_flag;
  return __all_sync(0xffffffffu, ok);
}

struct SegPos {
  int box, k, c16;  // int8 box (0, 1), row 0..63, 16-column group 0..7
};

__device__ __forceinline__ SegPos seg_pos(int seg) {
  const int g = seg & 511;
  const int i = g & 7;
  return {seg >> 9, 2 * (g >> 4) + (i >> 2), i ^ (((g >> 3) & 1) << 2)};
}

// Sixteen int8 weights of segment `sp` (row k, columns 16*c16 .. +15 of box b)
// -> fp16, stored into the weight tile: box b covers fp16 chunks 2b and 2b+1.
__device__ __forceinline__ void convert_store_segment(uint4 src, uint8_t* wtile, SegPos sp) {
  const int col = sp.c16 * 16;        // 0..112
  const int chunk = sp.box * 2 + (col >> 6);
  const int u = (col & 63) >> 3;      // 16-B unit of the fp16 row (even)
  uint32_t o[8];
  i8x4_to_f16x4(src.x, o[0], o[1]);
  i8x4_to_f16x4(src.y, o[2], o[3]);
  i8x4_to_f16x4(src.z, o[4], o[5]);
  i8x4_to_f16x4(src.w, o[6], o[7]);
  uint8_t* rowp = wtile + chunk * WCHUNK + sp.k * 128;
  *reinterpret_cast<uint4*>(rowp + ((u ^ (sp.k & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
  *reinterpret_cast<uint4*>(rowp + (((u + 1) ^ (sp.k & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
}

// Same, reading the segment from an int8 staging area of [64 K][128 N] boxes.
__device__ __forceinline__ void convert_int8_segment(const uint8_t* w8, uint8_t* wtile, int seg) {
  const SegPos sp = seg_pos(seg);
  const uint4 src = *reinterpret_cast<const uint4*>(w8 + sp.box * (BK * 128) + sp.k * 128 + sp.c16 * 16);
  convert_store_segment(src, wtile, sp);
}

// ---- combine in the down-projection epilogue ----------------------------
// Token t's output row is the sum of 2 * splits gate-scaled fp32 pieces: one
// per (slot, K split), each produced by a different tile (the two slots are
// different experts). Every piece is stored in Y[split, permuted row] by the
// epilogue that produced it, which then counts itself on the arrival counter
// of (t, column tile) with a release-acquire atomic add. The epilogue whose
// arrival completes the count (it never waits: everything it needs is already
// in memory) sums the pieces in a fixed order, slot 0 over splits, then slot 1
// over splits, then the two, adds the residual row if any, and stores the bf16
// output: the result does not depend on which tile finished last, and no
// output is updated with atomics. The pieces are dead once summed, so their L2
// lines are dropped without being written back to DRAM.

// Counter add with release (this thread's piece is visible device-wide before
// the count) and acquire (the pieces counted before are visible after it).
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Invalidate one 128-byte L2 line without writing it back (its data is dead).
__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// Fixed-order sum of the 2 * splits pieces of token `tok`, columns n0 + 8 * lane
// .. + 7, read from L2 (other SMs wrote them), stored as bf16.
__device__ __forceinline__ void combine_columns(const Params& p, int tok, int n0, int lane) {
  const int64_t p0 = p.slot_pos[2 * static_cast<int64_t>(tok)];
  const int64_t p1 = p.slot_pos[2 * static_cast<int64_t>(tok) + 1];
  if (kDebugBounds && !(index_ok(p0, p.rows) && index_ok(p1, p.rows))) {
    if (lane == 0) atomicOr(p.status, kStatusBounds);
    return;
  }
  const int64_t c = n0 + 8 * lane;
  const float* y = static_cast<const float*>(p.out);
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = b[j] = 0.0f;
  for (int s = 0; s < p.splits; ++s) {
    const float4* r0 = reinterpret_cast<const float4*>(y + s * p.split_stride + p0 * p.N + c);
    const float4* r1 = reinterpret_cast<const float4*>(y + s * p.split_stride + p1 * p.N + c);
    const float4 u0 = __ldcg(r0), u1 = __ldcg(r0 + 1), v0 = __ldcg(r1), v1 = __ldcg(r1 + 1);
    a[0] += u0.x; a[1] += u0.y; a[2] += u0.z; a[3] += u0.w;
    a[4] += u1.x; a[5] += u1.y; a[6] += u1.z; a[7] += u1.w;
    b[0] += v0.x; b[1] += v0.y; b[2] += v0.z; b[3] += v0.w;
    b[4] += v1.x; b[5] += v1.y; b[6] += v1.z; b[7] += v1.w;
  }
  float o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j] = a[j] + b[j];
  const int64_t at = static_cast<int64_t>(tok) * p.N + c;
  if (p.residual != nullptr) {
    const uint4 r = *reinterpret_cast<const uint4*>(p.residual + at);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] += __uint_as_float(w[j] << 16);
      o[2 * j + 1] += __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
  *reinterpret_cast<uint4*>(p.combine_out + at) =
      make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
  // Every lane has its values (they were summed above); then one lane per
  // 128-byte line drops the line: four lanes read 32 bytes each of it.
  __syncwarp();
  if ((lane & 3) == 0) {
    for (int s = 0; s < p.splits; ++s) {
      discard_l2_line(y + s * p.split_stride + p0 * p.N + c);
      discard_l2_line(y + s * p.split_stride + p1 * p.N + c);
    }
  }
}

// Called by a whole epilogue warp after each lane stored its row's piece of
// this tile (valid rows only). Lanes whose arrival completes a token's count
// hand the token to the warp, which combines one token row per pass with
// coalesced 1 KB reads.
__device__ __forceinline__ void combine_arrive(const Params& p, const Tile& t, int64_t row, bool valid) {
  int tok = 0;
  bool last = false;
  if (valid) {
    tok = p.perm_token[row];
    if (kDebugBounds && !index_ok(tok, p.rows / 2)) {
      atomicOr(p.status, kStatusBounds);
      valid = false;
      tok = 0;
    }
  }
  if (valid) {
    const int old =
        atomic_add_acq_rel_gpu(&p.combine_count[static_cast<int64_t>(tok) * (p.N / 256) + t.n0 / 256], 1);
    last = old == 2 * p.splits - 1;
  }
  unsigned m = __ballot_sync(0xffffffffu, last);
  if (m == 0) return;
  // Warp barrier: what the acquiring lanes observed is visible to every lane
  // that reads the pieces below.
  __syncwarp();
  const int lane = threadIdx.x % 32;
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    combine_columns(p, __shfl_sync(0xffffffffu, tok, src), t.n0, lane);
  }
}

// Weight-stream form of the same combine. There an epilogue warp q holds
// output columns n0 + 32q + lane and n0 + 128 + 32q + lane of every token row of
// the tile, so the meeting point is per (token, 256-column tile, warp): each
// warp counts its own 64 columns of a token and the arrival that completes that
// count (2 * splits pieces) sums them. No warp waits for another.
__device__ __forceinline__ void ws_combine_token(const Params& p, int tok, int n0, int q, int lane) {
  const int64_t p0 = p.slot_pos[2 * static_cast<int64_t>(tok)];
  const int64_t p1 = p.slot_pos[2 * static_cast<int64_t>(tok) + 1];
  if (kDebugBounds && !(index_ok(p0, p.rows) && index_ok(p1, p.rows))) {
    if (lane == 0) atomicOr(p.status, kStatusBounds);
    return;
  }
  const float* y = static_cast<const float*>(p.out);
  const int64_t ca = n0 + 32 * q + lane, cb = ca + 128;
  float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;  // slot 0 / slot 1, columns ca / cb
  for (int s = 0; s < p.splits; ++s) {
    const float* r0 = y + s * p.split_stride + p0 * p.N;
    const float* r1 = y + s * p.split_stride + p1 * p.N;
    a0 += __ldcg(r0 + ca);
    a1 += __ldcg(r0 + cb);
    b0 += __ldcg(r1 + ca);
    b1 += __ldcg(r1 + cb);
  }
  float oa = a0 + b0, ob = a1 + b1;
  const int64_t at = static_cast<int64_t>(tok) * p.N;
  if (p.residual != nullptr) {
    oa += __bfloat162float(p.residual[at + ca]);
    ob += __bfloat162float(p.residual[at + cb]);
  }
  p.combine_out[at + ca] = __float2bfloat16_rn(oa);
  p.combine_out[at + cb] = __float2bfloat16_rn(ob);
  __syncwarp();
  if (lane == 0) {  // this warp's two 128-byte lines of every piece are dead
    for (int s = 0; s < p.splits; ++s) {
      const float* r0 = y + s * p.split_stride + p0 * p.N;
      const float* r1 = y + s * p.split_stride + p1 * p.N;
      discard_l2_line(r0 + n0 + 32 * q);
      discard_l2_line(r0 + n0 + 128 + 32 * q);
      discard_l2_line(r1 + n0 + 32 * q);
      discard_l2_line(r1 + n0 + 128 + 32 * q);
    }
  }
}

// Called by a whole weight-stream epilogue warp after its lanes stored their
// columns of every row of the tile (rows t.row0 .. t.row0 + t.rows - 1).
__device__ __forceinline__ void ws_combine_arrive(const Params& p, const Tile& t, int q, int lane) {
  __threadfence();  // every lane's pieces are visible device-wide before any row is counted
  __syncwarp();
  const int64_t per_tok = static_cast<int64_t>(p.N / 256) * 4;
  for (int r0 = 0; r0 < t.rows; r0 += 32) {
    const int r = r0 + lane;
    int tok = 0;
    bool last = false;
    if (r < t.rows) {
      tok = p.perm_token[t.row0 + r];
      bool ok = true;
      if (kDebugBounds && !index_ok(tok, p.rows / 2)) {
        atomicOr(p.status, kStatusBounds);
        ok = false;
      }
      if (ok) {
        const int old = atomic_add_acq_rel_gpu(&p.combine_count[tok * per_tok + (t.n0 / 256) * 4 + q], 1);
        last = old == 2 * p.splits - 1;
      }
    }
    unsigned m = __ballot_sync(0xffffffffu, last);
    if (m == 0) continue;
    __syncwarp();
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      ws_combine_token(p, __shfl_sync(0xffffffffu, tok, src), t.n0, q, lane);
    }
  }
}

// Token-tile epilogue of one epilogue warp: TMEM lane = token row r (0..127 of
// this CTA's rows starting at permuted row `row_base`), 256 accumulator
// columns. GATEUP: columns 0..127 gate, 128..255 up -> H[row, n0 + c] (bf16; fp16 with int8 weights).
// DOWN: 256 output columns -> fp32 Y[split, row, n0 + c] = acc * gate[row],
// then (combine_count set) the combine above.
// GATEUP: H columns [c_begin, c_end) of the tile (a warp may take part of
// them); CW columns per TMEM load: 16 where the kernel runs 640 threads (at
// most 96 registers each), 32 otherwise.
template <int KIND, bool W8, int CW = (W8 ? 16 : 32)>
__device__ __forceinline__ void epilogue_token_rows(const Params& p, const Tile& t, uint32_t tbase, int r,
                                                    int64_t row_base, int nvalid, int c_begin = 0, int c_end = 128) {
  const bool valid = r < nvalid;
  const int64_t row = row_base + r;
  if (KIND == GATEUP) {
    static_assert(CW == 16 || CW == 32, "16 or 32 columns per TMEM load");
    uint16_t* hout = static_cast<uint16_t*>(p.out);
    uint32_t f16_bad = 0;  // int8 weights: an H value beyond the fp16 range
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += CW) {
      // int8 weights: the chunk's gate and up channel scales as 16-byte loads
      // (the same addresses in every lane), issued before the TMEM load so
      // that their latency overlaps it.
      uint32_t sg[CW / 2], su[CW / 2];
      if (W8) {
        const int64_t sc = static_cast<int64_t>(t.e) * p.N + t.n0 + c;
        const uint4* a = reinterpret_cast<const uint4*>(p.s0 + sc);
        const uint4* b = reinterpret_cast<const uint4*>(p.s1 + sc);
#pragma unroll
        for (int v = 0; v < CW / 8; ++v) {
          const uint4 x = __ldg(a + v), y = __ldg(b + v);
          sg[4 * v] = x.x; sg[4 * v + 1] = x.y; sg[4 * v + 2] = x.z; sg[4 * v + 3] = x.w;
          su[4 * v] = y.x; su[4 * v + 1] = y.y; su[4 * v + 2] = y.z; su[4 * v + 3] = y.w;
        }
      }
      uint32_t g[CW], u[CW];
      if constexpr (CW == 16) tmem_ld16x2(tbase + c, tbase + 128 + c, g, u);
      else tmem_ld32x2(tbase + c, tbase + 128 + c, g, u);
      uint32_t packed[CW / 2];
#pragma unroll
      for (int j = 0; j < CW; j += 2) {
        float g0 = __uint_as_float(g[j]), g1 = __uint_as_float(g[j + 1]);
        float u0 = __uint_as_float(u[j]), u1 = __uint_as_float(u[j + 1]);
        if (W8) {  // bf16 pair (lo = column j, hi = j + 1) -> fp32 by a shift
          g0 *= __uint_as_float(sg[j / 2] << 16);
          g1 *= __uint_as_float(sg[j / 2] & 0xFFFF0000u);
          u0 *= __uint_as_float(su[j / 2] << 16);
          u1 *= __uint_as_float(su[j / 2] & 0xFFFF0000u);
        }
        // int8 weights run the MMAs on fp16 operands, so H is stored as fp16 there.
        const float h0 = act_f32(g0, p.act) * u0, h1 = act_f32(g1, p.act) * u1;
        packed[j / 2] = W8 ? pack_f16x2(h0, h1) : pack_bf16x2(h0, h1);
        if (W8) f16_bad |= f16x2_nonfinite(packed[j / 2]);
      }
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(hout + row * p.N + t.n0 + c);
#pragma unroll
        for (int v = 0; v < CW / 8; ++v)
          dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
    }
    if (W8 && valid && f16_bad) atomicOr(p.status, kStatusFp16Range);
  } else {
    float* yout = static_cast<float*>(p.out) + static_cast<int64_t>(t.kb0 / p.kb_per_split) * p.split_stride;
    const float gate = valid ? p.gate_perm[row] : 0.0f;
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
      uint32_t sd[16];  // int8 weights: the chunk's 32 channel scales (four 16-byte loads)
      if (W8) {
        const uint4* a = reinterpret_cast<const uint4*>(p.s0 + static_cast<int64_t>(t.e) * p.N + t.n0 + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 x = __ldg(a + q);
          sd[4 * q] = x.x; sd[4 * q + 1] = x.y; sd[4 * q + 2] = x.z; sd[4 * q + 3] = x.w;
        }
      }
      uint32_t v[32];
      tmem_ld32(tbase + c, v);
      if (valid) {
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float a = __uint_as_float(v[j]);
          if (W8) a *= __uint_as_float((j & 1) ? (sd[j / 2] & 0xFFFF0000u) : (sd[j / 2] << 16));
          o[j] = a * gate;
        }
        float4* dst = reinterpret_cast<float4*>(yout + row * p.N + t.n0 + c);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
      }
    }
    if (p.combine_count != nullptr) combine_arrive(p, t, row, valid);
  }
}

}  // namespace tc
}  // namespace moe
