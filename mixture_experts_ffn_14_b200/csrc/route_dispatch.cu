// route_dispatch.cu — the CUDA-core stages around the expert GEMMs:
//   router   : fp32 logits x . w_router (+bias), softmax and top-2 per token
//              (grok-field-guide "Grok-1 blueprint", section "MoE sublayer";
//              Grok-1 book ch. 10, section 10.3.1: softmax over all experts,
//              top-k of the probabilities, gates not renormalised)
//   dispatch : counts, offsets and the stable (expert, token) permutation of
//              token slots, plus the gather of x rows into expert-contiguous
//              order; integer and deterministic (no capacity, no drop: ch. 10,
//              section 10.3.2)
//   combine  : out[t] = (gate-weighted slot-0 rows) + (slot-1 rows), summing the
//              split-K partials in a fixed order; no atomics on the output;
//              optionally followed by the post-RMSNorm and the residual add
//              (sandwich norm: ch. 10, section 10.3.1)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kTokPerWarp = kRouteTokens / (kRouterThreads / 32);  // 4
constexpr int kWrRows = 1024;  // router-weight rows staged in shared memory at a time

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The warp sums of 32 values at once, lane L receiving the sum of value L
// (v[j][e], L = j * kE + e): at each xor step a lane keeps the half of its
// values that its side of the pairing owns and adds the partner's copy of them,
// 31 shuffles instead of 5 per value. The pairings are warp_sum's, so every sum
// has the same bits as warp_sum of that value.
__device__ __forceinline__ float warp_reduce_scatter(const float (&v)[kTokPerWarp][kE], int lane) {
  static_assert(kTokPerWarp * kE == 32, "32 values");
  float a[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) a[i] = v[i / kE][i % kE];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? a[i] : a[i + off];
      const float keep = upper ? a[i + off] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return a[0];
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename TX>
struct Vec;  // 16-byte vector of activations

template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4 a, float (&v)[4]) {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
  }
  __device__ static void load(const float* p, float (&v)[4]) { unpack(*reinterpret_cast<const uint4*>(p), v); }
};

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4 a, float (&v)[8]) {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), v);
  }
};

struct Top2 {
  int e0, e1;
  float g0, g1;
};

// Top-2 of the 8 logits (strict comparisons keep the lower index on ties),
// softmax in fp32 and the gates (optionally renormalised).
__device__ __forceinline__ Top2 route_token(const float (&l)[kE], int32_t renormalize) {
  int e0 = 0;
  float m = l[0];
#pragma unroll
  for (int e = 1; e < kE; ++e)
    if (l[e] > m) {
      e0 = e;
      m = l[e];
    }
  int e1 = -1;
  float m1 = 0.0f;
#pragma unroll
  for (int e = 0; e < kE; ++e)
    if (e != e0 && (e1 < 0 || l[e] > m1)) {
      e1 = e;
      m1 = l[e];
    }
  float s = 0.0f;
#pragma unroll
  for (int e = 0; e < kE; ++e) s += expf(l[e] - m);
  const float p1 = expf(m1 - m);
  if (renormalize)  // Mixtral: the two probabilities divided by their sum
    return Top2{e0, e1, 1.0f / (1.0f + p1), p1 / (1.0f + p1)};
  return Top2{e0, e1, 1.0f / s, p1 / s};
}

// route_token for token t: idx / gates stored, the block's expert counts raised.
__device__ __forceinline__ Top2 finalize_token(const float (&l)[kE], int64_t t, int32_t renormalize,
                                               int32_t* __restrict__ idx, float* __restrict__ gates, int* cnt) {
  const Top2 r = route_token(l, renormalize);
  idx[2 * t] = r.e0;
  idx[2 * t + 1] = r.e1;
  gates[2 * t] = r.g0;
  gates[2 * t + 1] = r.g1;
  atomicAdd(&cnt[r.e0], 1);
  atomicAdd(&cnt[r.e1], 1);
  return r;
}

// Grid (token blocks of 32, d slices). One warp = 4 tokens; lanes split the CTA's
// slice of the hidden dimension in 16-byte vectors, the four tokens' loads
// issued together. With one slice the CTA finishes its tokens from registers.
// With several, each CTA stores its partial logits; the CTA that finds itself
// last for its token block (atomic counter, no waiting) sums the partials in
// slice order (so the result does not depend on arrival order) and finishes.
// Writes idx/gates per token and the block's per-expert slot count.
template <typename TX>
__global__ void __launch_bounds__(kRouterThreads) moe_router_kernel(
    const TX* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ bias, int64_t T, int64_t d,
    int32_t renormalize, int32_t slices, float* __restrict__ partial, int32_t* __restrict__ arrivals,
    int32_t* __restrict__ idx, float* __restrict__ gates, int32_t* __restrict__ hist) {
  constexpr int V = Vec<TX>::N;
  __shared__ int cnt[kE];
  __shared__ int last;
  __shared__ float4 wsm[(kWrRows * kE + (kWrRows / 4) * 4) / 4];
  if (threadIdx.x < kE) cnt[threadIdx.x] = 0;
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t blk = blockIdx.x;
  const int64_t t0 = blk * kRouteTokens + warp * kTokPerWarp;
  const int64_t len = d / slices;
  const int64_t c_begin = static_cast<int64_t>(blockIdx.y) * len;
  const TX* rows[kTokPerWarp];
#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j) rows[j] = x + min(t0 + j, T - 1) * d;  // clamped: always in bounds
  float acc[kTokPerWarp][kE];
#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[j][e] = 0.0f;

  // The slice's router weights pass through shared memory in chunks of
  // kWrRows rows, loaded with coalesced 16-byte reads. A lane then needs rows
  // base + V*lane + i: in global memory those sit 32*V bytes apart per lane (one
  // sector per lane per load); in shared memory each group of V rows is followed
  // by 16 bytes of padding, which spreads the lanes' 16-byte reads over all banks.
  for (int64_t cc = c_begin; cc < c_begin + len; cc += kWrRows) {
    const int rows_here = static_cast<int>(min(static_cast<int64_t>(kWrRows), c_begin + len - cc));
    __syncthreads();
    constexpr int kIt = 4;  // loads issued together before their stores
    for (int q0 = threadIdx.x; q0 < rows_here * 2; q0 += kIt * kRouterThreads) {
      float4 wv[kIt];
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int q = q0 + k * kRouterThreads;
        if (q < rows_here * 2) wv[k] = *reinterpret_cast<const float4*>(wr + (cc + (q >> 1)) * kE + (q & 1) * 4);
      }
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int q = q0 + k * kRouterThreads;
        const int r = q >> 1;
        if (q < rows_here * 2) wsm[(r * kE + (r / V) * 4 + (q & 1) * 4) / 4] = wv[k];
      }
    }
    __syncthreads();
#pragma unroll 2
    for (int r0 = lane * V; r0 < rows_here; r0 += 32 * V) {
      float xv[kTokPerWarp][V];
#pragma unroll
      for (int j = 0; j < kTokPerWarp; ++j) Vec<TX>::load(rows[j] + cc + r0, xv[j]);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int r = r0 + i;
        const float4 a = wsm[(r * kE + (r / V) * 4) / 4];
        const float4 b = wsm[(r * kE + (r / V) * 4) / 4 + 1];
        const float w[kE] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
          for (int e = 0; e < kE; ++e) acc[j][e] = fmaf(xv[j][i], w[e], acc[j][e]);
      }
    }
  }
  // lane L: the warp's sum for token t0 + L / 8, expert L % 8
  const float sum_l = warp_reduce_scatter(acc, lane);

  if (slices == 1) {
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j) {
      float l[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) l[e] = __shfl_sync(0xffffffffu, sum_l, j * kE + e) + (bias ? bias[e] : 0.0f);
      if (lane == j && t0 + j < T) finalize_token(l, t0 + j, renormalize, idx, gates, cnt);
    }
  } else {
    if (t0 + lane / kE < T) partial[(static_cast<int64_t>(blockIdx.y) * T + t0 + lane / kE) * kE + lane % kE] = sum_l;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&arrivals[blk], 1) == slices - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int64_t t = blk * kRouteTokens + threadIdx.x;
    if (threadIdx.x < kRouteTokens && t < T) {
      float l[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) l[e] = bias ? bias[e] : 0.0f;
      float sum[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) sum[e] = 0.0f;
      for (int sl = 0; sl < slices; ++sl) {
        const float* src = partial + (static_cast<int64_t>(sl) * T + t) * kE;
        const float4 a = __ldcg(reinterpret_cast<const float4*>(src));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(src + 4));
        sum[0] += a.x; sum[1] += a.y; sum[2] += a.z; sum[3] += a.w;
        sum[4] += b.x; sum[5] += b.y; sum[6] += b.z; sum[7] += b.w;
      }
#pragma unroll
      for (int e = 0; e < kE; ++e) l[e] += sum[e];
      finalize_token(l, t, renormalize, idx, gates, cnt);
    }
  }
  __syncthreads();
  if (threadIdx.x < kE) hist[blk * kE + threadIdx.x] = cnt[threadIdx.x];
}

// Exclusive prefix over router blocks of the per-block expert histograms, and
// their totals, for batches with many blocks (one CTA of 1024 threads: thread i
// owns a contiguous run of blocks, sums it, the CTA scans the 1024 run sums per
// expert, and each thread writes its run's prefixes). Linear in the blocks, so
// the dispatch CTAs read their offsets instead of summing all predecessors.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) moe_hist_scan_kernel(const int32_t* __restrict__ hist, int64_t nblk,
                                                                     int32_t* __restrict__ pre,
                                                                     int32_t* __restrict__ tot) {
  __shared__ int wsum[kE][kScanThreads / 32];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t per = (nblk + kScanThreads - 1) / kScanThreads;
  const int64_t b0 = min(nblk, tid * per), b1 = min(nblk, b0 + per);
  int run[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) run[e] = 0;
  for (int64_t b = b0; b < b1; ++b) {
    const int4 lo = *reinterpret_cast<const int4*>(hist + b * kE);
    const int4 hi = *reinterpret_cast<const int4*>(hist + b * kE + 4);
    run[0] += lo.x; run[1] += lo.y; run[2] += lo.z; run[3] += lo.w;
    run[4] += hi.x; run[5] += hi.y; run[6] += hi.z; run[7] += hi.w;
  }
  // Exclusive scan of the run sums over the CTA, per expert.
  int excl[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    int v = run[e];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    excl[e] = v - run[e];                       // exclusive within the warp
    if (lane == 31) wsum[e][warp] = v;          // warp total
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const int w = wsum[e][lane];
      int v = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      wsum[e][lane] = v - w;                    // exclusive over warps
      if (lane == 31) tot[e] = v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < kE; ++e) excl[e] += wsum[e][warp];
  for (int64_t b = b0; b < b1; ++b) {
    const int4 lo = *reinterpret_cast<const int4*>(hist + b * kE);
    const int4 hi = *reinterpret_cast<const int4*>(hist + b * kE + 4);
    *reinterpret_cast<int4*>(pre + b * kE) = make_int4(excl[0], excl[1], excl[2], excl[3]);
    *reinterpret_cast<int4*>(pre + b * kE + 4) = make_int4(excl[4], excl[5], excl[6], excl[7]);
    excl[0] += lo.x; excl[1] += lo.y; excl[2] += lo.z; excl[3] += lo.w;
    excl[4] += hi.x; excl[5] += hi.y; excl[6] += hi.z; excl[7] += hi.w;
  }
}

// Eight bf16 (one 16-byte vector) -> eight fp16, round to nearest even.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(__uint_as_float(w << 16)));
  return r;
}
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
}
// Nonzero if one of the eight fp16 values is infinite or NaN (exponent field
// all ones): a bf16 input of magnitude above 65504 overflowed in the conversion.
__device__ __forceinline__ uint32_t f16x8_nonfinite(uint4 h) {
  uint32_t bad = 0;
  const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    bad |= static_cast<uint32_t>((w[i] & 0x7C00u) == 0x7C00u) | static_cast<uint32_t>((w[i] & 0x7C000000u) == 0x7C000000u);
  return bad;
}

// Same 32-token range per CTA as the router. Each CTA sums the per-CTA
// histograms to find where its tokens land (no cross-CTA waiting), ranks its
// tokens per expert with warp ballots (token order = stable), writes the
// permutation arrays and copies the x rows to their permuted positions.
// F16: the copy converts bf16 rows to fp16 (round to nearest even), for the
// int8-weight GEMMs, whose MMAs run on fp16 operands.
template <typename TX, bool F16 = false>
__global__ void __launch_bounds__(256) moe_dispatch_kernel(
    const TX* __restrict__ x, int64_t T, int64_t d, int64_t nblk, const int32_t* __restrict__ idx,
    const float* __restrict__ gates, const int32_t* __restrict__ hist, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token, int32_t* __restrict__ perm_slot,
    int32_t* __restrict__ slot_pos, float* __restrict__ gate_perm, TX* __restrict__ xp,
    const int32_t* __restrict__ hist_pre, const int32_t* __restrict__ hist_tot, uint32_t* __restrict__ status) {
  // blockIdx.y splits the row gather of the block across gridDim.y CTAs; all of
  // them rank the block's tokens (cheap), the first one writes the permutation.
  __shared__ int red[8][2 * kE];
  __shared__ int base[kE];
  __shared__ int pos_sm[kRouteTokens][2];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t blk = blockIdx.x;

  // This block's slots start, per expert, after those of all earlier blocks:
  // read from the scan (many blocks) or summed here (few blocks, no extra launch).
  int tot[kE], pre[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) tot[e] = pre[e] = 0;
  if (hist_pre != nullptr) {
    if (threadIdx.x == 0) {
#pragma unroll
      for (int e = 0; e < kE; ++e) {
        tot[e] = hist_tot[e];
        pre[e] = hist_pre[blk * kE + e];
      }
    }
  } else {
    for (int64_t c = threadIdx.x; c < nblk; c += blockDim.x) {
#pragma unroll
      for (int e = 0; e < kE; ++e) {
        const int v = hist[c * kE + e];
        tot[e] += v;
        if (c < blk) pre[e] += v;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    tot[e] = warp_sum_i(tot[e]);
    pre[e] = warp_sum_i(pre[e]);
  }
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      red[warp][e] = tot[e];
      red[warp][kE + e] = pre[e];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int total[kE], before[kE];
    for (int e = 0; e < kE; ++e) {
      total[e] = before[e] = 0;
      for (int w = 0; w < 8; ++w) {
        total[e] += red[w][e];
        before[e] += red[w][kE + e];
      }
    }
    int off = 0;
    for (int e = 0; e < kE; ++e) {
      base[e] = off + before[e];
      if (blk == 0 && blockIdx.y == 0) {
        counts[e] = total[e];
        offsets[e] = off;
      }
      off += total[e];
    }
    if (blk == 0 && blockIdx.y == 0) offsets[kE] = off;
  }
  __syncthreads();

  if (warp == 0) {
    const int64_t t = blk * kRouteTokens + lane;
    const bool valid = t < T;
    const int a = valid ? idx[2 * t] : -1;
    const int b = valid ? idx[2 * t + 1] : -1;
    const unsigned lt = (1u << lane) - 1u;
    int pa = -1, pb = -1;
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const unsigned m = __ballot_sync(0xffffffffu, a == e || b == e);
      const int r = base[e] + __popc(m & lt);
      if (a == e) pa = r;
      if (b == e) pb = r;
    }
    bool ok = valid;
    if (kDebugBounds && valid && !(index_ok(pa, 2 * T) && index_ok(pb, 2 * T))) {
      atomicOr(status, kStatusBounds);  // an expert id outside [0, E): skip the token
      ok = false;
      pa = pb = -1;
    }
    if (ok && blockIdx.y == 0) {
      perm_token[pa] = static_cast<int32_t>(t);
      perm_slot[pa] = 0;
      perm_token[pb] = static_cast<int32_t>(t);
      perm_slot[pb] = 1;
      slot_pos[2 * t] = pa;
      slot_pos[2 * t + 1] = pb;
      gate_perm[pa] = gates[2 * t];
      gate_perm[pb] = gates[2 * t + 1];
    }
    pos_sm[lane][0] = pa;
    pos_sm[lane][1] = pb;
  }
  __syncthreads();
  if (xp == nullptr) return;  // the expert GEMM gathers the rows itself

  // Gather: 64 rows of d elements, as 16-byte vectors; eight loads in flight
  // per thread before their stores.
  const int64_t vec_per_row = d * static_cast<int64_t>(sizeof(TX)) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(xp);
  const int64_t total = 2 * kRouteTokens * vec_per_row;
  const int64_t stride = static_cast<int64_t>(blockDim.x) * gridDim.y;
  uint32_t f16_bad = 0;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; i0 < total; i0 += 8 * stride) {
    uint4 v[8];
    int64_t o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t i = i0 + u * stride;
      o[u] = -1;
      if (i < total) {
        const int r = static_cast<int>(i / vec_per_row);
        const int64_t c = i - r * vec_per_row;
        const int pos = pos_sm[r >> 1][r & 1];
        if (pos >= 0) {
          v[u] = src[(blk * kRouteTokens + (r >> 1)) * vec_per_row + c];
          o[u] = static_cast<int64_t>(pos) * vec_per_row + c;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (o[u] < 0) continue;
      if (F16) {
        const uint4 h = bf16x8_to_f16x8(v[u]);
        f16_bad |= f16x8_nonfinite(h);
        dst[o[u]] = h;
      } else {
        dst[o[u]] = v[u];
      }
    }
  }
  if (F16 && f16_bad) atomicOr(status, kStatusFp16Range);
}

// ---- small batches: router and dispatch in one cluster launch -------------
// For T <= kSmallMaxT (decode) the two stages above cost more in launches and
// global round trips (partial logits, an arrival counter, a second kernel)
// than in work. Here one cluster of kSmallCTAs CTAs does both:
//   1. CTA c forms the partial logits of every token over its slice of the
//      hidden dimension (d / kSmallCTAs elements; the slice's router weights
//      staged through shared memory as in the router kernel) and keeps them in
//      its shared memory;
//   2. cluster barrier; CTA 0 sums each token's partials in slice order
//      (reading the other CTAs' shared memory), finishes the routing exactly
//      as the router kernel does (same top-2, softmax and gate arithmetic) and
//      computes counts, offsets and the stable (expert, token) permutation;
//   3. cluster barrier; every CTA reads the positions it needs out of CTA 0's
//      shared memory, arrives on the cluster barrier and writes the permuted
//      rows of x (converted to fp16 for int8 weights). When one pass of the
//      warps covers the tokens (T <= 64) and a lane's share of the slice fits
//      kXU vectors, the x values loaded in step 1 are still in registers and
//      each CTA stores its slice of both of a token's rows; otherwise the 2T
//      rows are read from x again, eight 16-byte loads in flight per thread;
//   4. wait on that barrier, so CTA 0's shared memory outlives those reads.
// The cluster has 16 CTAs (above the portable 8; small_route_dispatch checks
// once per device that it fits) because the loads and stores of steps 1 and 3
// are bound by what few SMs keep in flight: with 8 CTAs the kernel took 13 us
// at T = 64, d = 6144 on a B200, 3 us of it in the stores of step 3.
constexpr int kSmallCTAs = 16;  // a non-portable cluster size: checked per device before use
constexpr int kSmallMaxT = 128;
constexpr int kSmallThreads = 512;
constexpr int64_t kSmallMaxD = 65536;  // 2 * kSmallMaxT rows of d elements index in 32 bits
constexpr int kXU = 2;                 // 16-byte x vectors per lane and token loaded together
constexpr int kStageIt = (2 * kWrRows + kSmallThreads - 1) / kSmallThreads;  // router-row float4 per thread

template <typename TX, bool F16 = false>
__global__ void __launch_bounds__(kSmallThreads)
    moe_route_dispatch_small_kernel(const TX* __restrict__ x, const float* __restrict__ wr,
                                    const float* __restrict__ bias, int64_t T, int64_t d, int32_t renormalize,
                                    int32_t* __restrict__ idx, float* __restrict__ gates,
                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                    int32_t* __restrict__ perm_token, int32_t* __restrict__ perm_slot,
                                    int32_t* __restrict__ slot_pos, float* __restrict__ gate_perm,
                                    TX* __restrict__ xp, uint32_t* __restrict__ status) {
  using namespace moe::sm100;
  constexpr int V = Vec<TX>::N;
  __shared__ __align__(16) float part[kSmallMaxT][kE];  // this CTA's partial logits
  __shared__ int sel[kSmallMaxT][2];      // CTA 0: chosen experts
  __shared__ float sgate[kSmallMaxT][2];  // CTA 0: their gates
  __shared__ int pos[kSmallMaxT][2];      // CTA 0: permuted row of each (token, slot)
  __shared__ int cnt[kE];
  __shared__ float4 wsm[(kWrRows * kE + (kWrRows / 4) * 4) / 4];
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kWarps = kSmallThreads / 32;
  if (threadIdx.x < kE) cnt[threadIdx.x] = 0;

  // 1. Partial logits over this CTA's slice, kTokPerWarp tokens per warp pass.
  //    Each lane issues its kXU x vectors of every token before the router
  //    rows are staged, so the two loads overlap.
  const int64_t len = d / kSmallCTAs;
  const int64_t c_begin = static_cast<int64_t>(rank) * len;
  // One pass over the tokens and one block of x vectors: the x values stay in
  // registers for the copy in step 3 (decode shapes: T <= 64, d <= 6144 bf16).
  const bool keep = T <= kWarps * kTokPerWarp && len <= kWrRows && len <= static_cast<int64_t>(kXU) * 32 * V;
  uint4 raw[kXU][kTokPerWarp];
  int64_t staged = -1;  // the slice chunk whose router rows wsm holds (the same in every thread)
  for (int64_t tb = static_cast<int64_t>(warp) * kTokPerWarp; tb < kSmallMaxT; tb += kWarps * kTokPerWarp) {
    // every warp runs the same number of passes (the __syncthreads below)
    const TX* rows[kTokPerWarp];
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j) rows[j] = x + min(tb + j, T - 1) * d;  // clamped: always in bounds
    float acc[kTokPerWarp][kE];
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
      for (int e = 0; e < kE; ++e) acc[j][e] = 0.0f;
    for (int64_t cc = c_begin; cc < c_begin + len; cc += kWrRows) {
      const int rows_here = static_cast<int>(min(static_cast<int64_t>(kWrRows), c_begin + len - cc));
      for (int xb = 0; xb < rows_here; xb += kXU * 32 * V) {
        if (tb < T) {
#pragma unroll
          for (int u = 0; u < kXU; ++u) {
            const int r0 = xb + (u * 32 + lane) * V;
            if (r0 < rows_here)
#pragma unroll
              for (int j = 0; j < kTokPerWarp; ++j) raw[u][j] = *reinterpret_cast<const uint4*>(rows[j] + cc + r0);
          }
        }
        if (cc != staged) {  // a slice within kWrRows rows is staged once for all passes
          float4 wv[kStageIt];  // every load issued before the first store
#pragma unroll
          for (int k = 0; k < kStageIt; ++k) {
            const int q = threadIdx.x + k * kSmallThreads;
            if (q < rows_here * 2) wv[k] = *reinterpret_cast<const float4*>(wr + (cc + (q >> 1)) * kE + (q & 1) * 4);
          }
          __syncthreads();
#pragma unroll
          for (int k = 0; k < kStageIt; ++k) {
            const int q = threadIdx.x + k * kSmallThreads;
            const int r = q >> 1;
            if (q < rows_here * 2) wsm[(r * kE + (r / V) * 4 + (q & 1) * 4) / 4] = wv[k];
          }
          __syncthreads();
          staged = cc;
        }
        if (tb < T) {
#pragma unroll
          for (int u = 0; u < kXU; ++u) {
            const int r0 = xb + (u * 32 + lane) * V;
            if (r0 < rows_here) {
              float xv[kTokPerWarp][V];
#pragma unroll
              for (int j = 0; j < kTokPerWarp; ++j) Vec<TX>::unpack(raw[u][j], xv[j]);
#pragma unroll
              for (int i = 0; i < V; ++i) {
                const int r = r0 + i;
                const float4 a = wsm[(r * kE + (r / V) * 4) / 4];
                const float4 b = wsm[(r * kE + (r / V) * 4) / 4 + 1];
                const float w[kE] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
                  for (int e = 0; e < kE; ++e) acc[j][e] = fmaf(xv[j][i], w[e], acc[j][e]);
              }
            }
          }
        }
      }
    }
    if (tb < T) {
      // lane L: the warp's sum for token tb + L / 8, expert L % 8
      static_assert(kTokPerWarp * kE == 32, "one (token, expert) value per lane");
      part[tb + lane / kE][lane % kE] = warp_reduce_scatter(acc, lane);
    }
  }
  cluster_sync();

  // 2. CTA 0: routing and the permutation. Four threads per token each sum
  //    a quarter of the CTAs' partials (in CTA order); the quarters are added
  //    as (q0 + q1) + (q2 + q3), the same in all four lanes.
  if (rank == 0) {
    static_assert(kSmallThreads == 4 * kSmallMaxT && kSmallCTAs % 4 == 0, "four threads per token");
    constexpr int kPer = kSmallCTAs / 4;
    const int t = threadIdx.x >> 2, q = threadIdx.x & 3;
    float sum[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) sum[e] = 0.0f;
    if (t < T) {
      float4 pa[kPer], pb[kPer];
#pragma unroll
      for (int c = 0; c < kPer; ++c) {
        const uint32_t at = mapa_shared(&part[t][0], static_cast<uint32_t>(q * kPer + c));
        pa[c] = ld_shared_cluster_f32x4(at);
        pb[c] = ld_shared_cluster_f32x4(at + 16);
      }
#pragma unroll
      for (int c = 0; c < kPer; ++c) {
        sum[0] += pa[c].x; sum[1] += pa[c].y; sum[2] += pa[c].z; sum[3] += pa[c].w;
        sum[4] += pb[c].x; sum[5] += pb[c].y; sum[6] += pb[c].z; sum[7] += pb[c].w;
      }
    }
#pragma unroll
    for (int e = 0; e < kE; ++e) sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], 1);
#pragma unroll
    for (int e = 0; e < kE; ++e) sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], 2);
    if (t < T && q == 0) {
      float l[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) l[e] = (bias ? bias[e] : 0.0f) + sum[e];
      const Top2 r = route_token(l, renormalize);
      sel[t][0] = r.e0;
      sel[t][1] = r.e1;
      sgate[t][0] = r.g0;
      sgate[t][1] = r.g1;
      atomicAdd(&cnt[r.e0], 1);
      atomicAdd(&cnt[r.e1], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int base[kE];
      int off = 0;
#pragma unroll
      for (int e = 0; e < kE; ++e) {
        base[e] = off;
        off += cnt[e];
      }
      const unsigned lt = (1u << lane) - 1u;
      for (int t0 = 0; t0 < T; t0 += 32) {
        const int t = t0 + lane;
        const bool valid = t < T;
        const int a = valid ? sel[t][0] : -1;
        const int b = valid ? sel[t][1] : -1;
        int pa = -1, pb = -1;
#pragma unroll
        for (int e = 0; e < kE; ++e) {
          const unsigned m = __ballot_sync(0xffffffffu, a == e || b == e);
          const int r = base[e] + __popc(m & lt);
          if (a == e) pa = r;
          if (b == e) pb = r;
          base[e] += __popc(m);
        }
        if (valid) {
          if (kDebugBounds && !(index_ok(pa, 2 * T) && index_ok(pb, 2 * T))) {
            atomicOr(status, kStatusBounds);
            pa = pb = -1;
          }
          pos[t][0] = pa;
          pos[t][1] = pb;
        }
      }
    }
  }
  cluster_sync();
  // CTA 0 stores the routing and the permutation to global memory now, off
  // the path to the barrier above (nothing in this kernel reads them back).
  if (rank == 0) {
    const int i = threadIdx.x;
    if (i < 2 * T) {
      const int t = i >> 1, s = i & 1;
      const int p = pos[t][s];
      idx[i] = sel[t][s];
      gates[i] = sgate[t][s];
      if (p >= 0) {
        slot_pos[i] = p;
        perm_token[p] = t;
        perm_slot[p] = s;
        gate_perm[p] = sgate[t][s];
      }
    }
    if (i < kE) {
      int base = 0;
      for (int e = 0; e < i; ++e) base += cnt[e];
      counts[i] = cnt[i];
      offsets[i] = base;
    }
    if (i == kE) offsets[kE] = static_cast<int32_t>(2 * T);
  }

  // 3. The permuted copy of x.
  uint32_t f16_bad = 0;
  if (keep) {
    // From registers: each warp stores its tokens' slice of x into both of
    // their permuted rows (positions read from CTA 0, lane l: token l/2, slot l%2).
    const int64_t tb = static_cast<int64_t>(warp) * kTokPerWarp;
    int p_lane = -1;
    if (lane < 2 * kTokPerWarp && tb + lane / 2 < T)
      p_lane = ld_shared_cluster_s32(mapa_shared(&pos[tb + lane / 2][lane & 1], 0));
    cluster_arrive();  // this CTA is done with CTA 0's shared memory
    uint4* dst = reinterpret_cast<uint4*>(xp);
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int p = __shfl_sync(0xffffffffu, p_lane, 2 * j + s);
        if (tb + j >= T || p < 0) continue;
#pragma unroll
        for (int u = 0; u < kXU; ++u) {
          const int r0 = (u * 32 + lane) * V;
          if (r0 >= len) continue;
          const int64_t at = (static_cast<int64_t>(p) * d + c_begin + r0) / V;  // 16-byte vector index
          if (F16) {
            const uint4 h = bf16x8_to_f16x8(raw[u][j]);
            f16_bad |= f16x8_nonfinite(h);
            dst[at] = h;
          } else {
            dst[at] = raw[u][j];
          }
        }
      }
    if (F16 && f16_bad) atomicOr(status, kStatusFp16Range);
    cluster_wait();  // CTA 0's shared memory stays until every CTA has read it
    return;
  }
  // Otherwise: positions into this CTA's shared memory, then the 2T rows as
  // 16-byte vectors read again from x, spread over all the cluster's threads.
  if (rank != 0)
    for (int i = threadIdx.x; i < 2 * T; i += blockDim.x)
      (&pos[0][0])[i] = ld_shared_cluster_s32(mapa_shared(&pos[0][0] + i, 0));
  cluster_arrive();  // this CTA is done with CTA 0's shared memory
  __syncthreads();
  // 32-bit indices: 2T * vec_per_row <= 2 * kSmallMaxT * kSmallMaxD / 4 < 2^31
  const int vec_per_row = static_cast<int>(d * static_cast<int64_t>(sizeof(TX)) / 16);
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(xp);
  const int total = 2 * static_cast<int>(T) * vec_per_row;
  constexpr int stride = kSmallCTAs * kSmallThreads;
  for (int i0 = static_cast<int>(rank) * kSmallThreads + threadIdx.x; i0 < total; i0 += 8 * stride) {
    uint4 v[8];
    int o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * stride;
      o[u] = -1;
      if (i < total) {
        const int r = i / vec_per_row;
        const int c = i - r * vec_per_row;
        const int p = pos[r >> 1][r & 1];
        if (p >= 0) {
          v[u] = src[(r >> 1) * vec_per_row + c];
          o[u] = p * vec_per_row + c;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (o[u] < 0) continue;
      if (F16) {
        const uint4 h = bf16x8_to_f16x8(v[u]);
        f16_bad |= f16x8_nonfinite(h);
        dst[o[u]] = h;
      } else {
        dst[o[u]] = v[u];
      }
    }
  }
  if (F16 && f16_bad) atomicOr(status, kStatusFp16Range);
  cluster_wait();  // CTA 0's shared memory stays until every CTA has read it
}

template <typename TO>
__device__ __forceinline__ void store4(TO* p, float4 v);

template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}

template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

template <typename TO>
__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ y, int64_t split_stride,
                                                          int32_t splits, const int32_t* __restrict__ slot_pos,
                                                          int64_t T, int64_t d, TO* __restrict__ out,
                                                          uint32_t* __restrict__ status) {
  const int64_t q = d / 4;
  const int64_t n = T * q;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // Four outputs per thread per pass, their loads issued before any store.
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n; i0 += 4 * stride) {
    float4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * stride;
      r[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < n) {
        const int64_t t = i / q;
        const int64_t c = (i - t * q) * 4;
        const int64_t p0 = slot_pos[2 * t], p1 = slot_pos[2 * t + 1];
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (kDebugBounds && !(index_ok(p0, 2 * T) && index_ok(p1, 2 * T))) {
          atomicOr(status, kStatusBounds);
          continue;
        }
        for (int s = 0; s < splits; ++s) {
          const float4 uu = *reinterpret_cast<const float4*>(y + s * split_stride + p0 * d + c);
          const float4 vv = *reinterpret_cast<const float4*>(y + s * split_stride + p1 * d + c);
          a.x += uu.x; a.y += uu.y; a.z += uu.z; a.w += uu.w;
          b.x += vv.x; b.y += vv.y; b.z += vv.z; b.w += vv.w;
        }
        r[u] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < n) {
        const int64_t t = i / q;
        store4<TO>(out + t * d + (i - t * q) * 4, r[u]);
      }
    }
  }
}

template <typename TO>
__device__ __forceinline__ float4 load4(const TO* p);

template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}

// Combine with the sublayer's post-RMSNorm and/or residual add: one CTA per
// token row. Pass 1 forms y = (slot-0 rows) + (slot-1 rows) in fp32 and its sum
// of squares (fixed reduction order: per-thread strided sums, then a fixed
// tree); pass 2 forms y again (its rows are now in L2) and writes
// residual + w * y * rsqrt(mean(y^2) + eps).
template <typename TO>
__global__ void __launch_bounds__(256) moe_combine_norm_kernel(const float* __restrict__ y, int64_t split_stride,
                                                               int32_t splits, const int32_t* __restrict__ slot_pos,
                                                               int64_t d, const TO* __restrict__ residual,
                                                               const float* __restrict__ norm_weight, float eps,
                                                               TO* __restrict__ out, uint32_t* __restrict__ status) {
  __shared__ float red[8];
  const int64_t t = blockIdx.x;
  const int64_t p0 = slot_pos[2 * t], p1 = slot_pos[2 * t + 1];
  if (kDebugBounds && !(index_ok(p0, 2 * static_cast<int64_t>(gridDim.x)) &&
                        index_ok(p1, 2 * static_cast<int64_t>(gridDim.x)))) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBounds);
    return;  // uniform over the CTA: one token row per CTA
  }
  auto row_y = [&](int64_t c) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int s = 0; s < splits; ++s) {
      const float4 u = *reinterpret_cast<const float4*>(y + s * split_stride + p0 * d + c);
      const float4 v = *reinterpret_cast<const float4*>(y + s * split_stride + p1 * d + c);
      a.x += u.x; a.y += u.y; a.z += u.z; a.w += u.w;
      b.x += v.x; b.y += v.y; b.z += v.z; b.w += v.w;
    }
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  };
  float scale = 1.0f;
  if (norm_weight) {
    float ss = 0.0f;
    for (int64_t c = 4 * threadIdx.x; c < d; c += 4 * blockDim.x) {
      const float4 v = row_y(c);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
      float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.0f;
      v = warp_sum(v);
      if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    scale = rsqrtf(red[0] / static_cast<float>(d) + eps);
  }
  for (int64_t c = 4 * threadIdx.x; c < d; c += 4 * blockDim.x) {
    float4 v = row_y(c);
    if (norm_weight) {
      const float4 w = *reinterpret_cast<const float4*>(norm_weight + c);
      v = make_float4(v.x * scale * w.x, v.y * scale * w.y, v.z * scale * w.z, v.w * scale * w.w);
    }
    if (residual) {
      const float4 r = load4<TO>(residual + t * d + c);
      v = make_float4(v.x + r.x, v.y + r.y, v.z + r.z, v.w + r.w);
    }
    store4<TO>(out + t * d + c, v);
  }
}

}  // namespace

int32_t router_slices(int64_t T, int64_t d, moe_dtype_t dtype) {
  // Split d so that about two CTAs per SM run; each slice a whole number of
  // 32-lane x 16-byte steps.
  const int64_t chunk = 32 * (dtype == MOE_F32 ? 4 : 8);
  const int64_t nchunks = d / chunk;
  const int64_t nblk = (T + kRouteTokens - 1) / kRouteTokens;
  int64_t s = std::min<int64_t>(nchunks, std::max<int64_t>(1, (2 * device_sm_count() + nblk - 1) / nblk));
  while (s > 1 && nchunks % s != 0) --s;
  return static_cast<int32_t>(std::max<int64_t>(1, s));
}

cudaError_t launch_router(moe_dtype_t dtype, const void* x, const float* w_router, const float* bias, int64_t T,
                          int64_t d, int32_t renormalize, int32_t slices, float* partial, int32_t* arrivals,
                          int32_t* idx, float* gates, int32_t* hist, cudaStream_t s) {
  const int64_t nblk = (T + kRouteTokens - 1) / kRouteTokens;
  const dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(slices), 1);
  if (dtype == MOE_F32)
    moe_router_kernel<float><<<grid, kRouterThreads, 0, s>>>(static_cast<const float*>(x), w_router, bias, T, d,
                                                             renormalize, slices, partial, arrivals, idx, gates,
                                                             hist);
  else
    moe_router_kernel<__nv_bfloat16><<<grid, kRouterThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), w_router, bias, T, d, renormalize, slices, partial, arrivals, idx,
        gates, hist);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(moe_dtype_t dtype, const void* x, int64_t T, int64_t d, int64_t nblk,
                            const int32_t* idx, const float* gates, const int32_t* hist, int32_t* hist_pre,
                            int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                            int32_t* slot_pos, float* gate_perm, void* xp, uint32_t* status, cudaStream_t s) {
  // Many router blocks: scan their histograms once (hist_pre holds nblk * E
  // prefixes followed by E totals); few: each dispatch CTA sums them itself.
  const int32_t* pre = nullptr;
  const int32_t* tot = nullptr;
  if (nblk > kDispatchSumBlocks) {
    moe_hist_scan_kernel<<<1, kScanThreads, 0, s>>>(hist, nblk, hist_pre, hist_pre + nblk * kE);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pre = hist_pre;
    tot = hist_pre + nblk * kE;
  }
  // Extra CTAs along y only split the row gather; without Xp one suffices.
  const int64_t g =
      xp ? std::min<int64_t>(16, std::max<int64_t>(1, (2 * device_sm_count() + nblk - 1) / nblk)) : 1;
  const dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(g), 1);
  if (dtype == MOE_F32)
    moe_dispatch_kernel<float><<<grid, 256, 0, s>>>(
        static_cast<const float*>(x), T, d, nblk, idx, gates, hist, counts, offsets, perm_token, perm_slot,
        slot_pos, gate_perm, static_cast<float*>(xp), pre, tot, status);
  else if (dtype == MOE_BF16_INT8W)
    moe_dispatch_kernel<__nv_bfloat16, true><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), T, d, nblk, idx, gates, hist, counts, offsets, perm_token,
        perm_slot, slot_pos, gate_perm, static_cast<__nv_bfloat16*>(xp), pre, tot, status);
  else
    moe_dispatch_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), T, d, nblk, idx, gates, hist, counts, offsets, perm_token,
        perm_slot, slot_pos, gate_perm, static_cast<__nv_bfloat16*>(xp), pre, tot, status);
  return cudaGetLastError();
}

namespace {

cudaLaunchConfig_t small_config(cudaLaunchAttribute* at, cudaStream_t s) {
  at->id = cudaLaunchAttributeClusterDimension;
  at->val.clusterDim.x = kSmallCTAs;
  at->val.clusterDim.y = 1;
  at->val.clusterDim.z = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(kSmallCTAs, 1, 1);
  c.blockDim = dim3(kSmallThreads, 1, 1);
  c.stream = s;
  c.attrs = at;
  c.numAttrs = 1;
  return c;
}

// Allows the cluster size above the portable 8 and checks that one cluster
// fits on this device; 0 when it does not (the two-kernel path is used then).
template <typename TX, bool F16>
int small_cluster_fits() {
  auto kern = moe_route_dispatch_small_kernel<TX, F16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute at;
  const cudaLaunchConfig_t c = small_config(&at, nullptr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &c) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n >= 1 ? 1 : 0;
}

template <typename TX, bool F16>
cudaError_t launch_small(const TX* x, const float* w_router, const float* bias, int64_t T, int64_t d,
                         int32_t renormalize, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets,
                         int32_t* perm_token, int32_t* perm_slot, int32_t* slot_pos, float* gate_perm, TX* xp,
                         uint32_t* status, cudaStream_t s) {
  cudaLaunchAttribute at;
  const cudaLaunchConfig_t c = small_config(&at, s);
  return cudaLaunchKernelEx(&c, moe_route_dispatch_small_kernel<TX, F16>, x, w_router, bias, T, d, renormalize,
                            idx, gates, counts, offsets, perm_token, perm_slot, slot_pos, gate_perm, xp, status);
}

}  // namespace

bool small_route_dispatch(int64_t T, int64_t d, const void* xp) {
  if (!(T > 0 && T <= kSmallMaxT && d <= kSmallMaxD && xp != nullptr)) return false;
  const int ok = once_per_device(reinterpret_cast<const void*>(&small_route_dispatch), [](const void*) -> int {
    return small_cluster_fits<float, false>() && small_cluster_fits<__nv_bfloat16, false>() &&
                   small_cluster_fits<__nv_bfloat16, true>()
               ? 1
               : 0;
  });
  return ok == 1;
}

cudaError_t launch_route_dispatch_small(moe_dtype_t dtype, const void* x, const float* w_router, const float* bias,
                                        int64_t T, int64_t d, int32_t renormalize, int32_t* idx, float* gates,
                                        int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                                        int32_t* slot_pos, float* gate_perm, void* xp, uint32_t* status,
                                        cudaStream_t s) {
  if (dtype == MOE_F32)
    return launch_small<float, false>(static_cast<const float*>(x), w_router, bias, T, d, renormalize, idx, gates,
                                      counts, offsets, perm_token, perm_slot, slot_pos, gate_perm,
                                      static_cast<float*>(xp), status, s);
  using B = __nv_bfloat16;
  if (dtype == MOE_BF16_INT8W)
    return launch_small<B, true>(static_cast<const B*>(x), w_router, bias, T, d, renormalize, idx, gates, counts,
                                 offsets, perm_token, perm_slot, slot_pos, gate_perm, static_cast<B*>(xp), status, s);
  return launch_small<B, false>(static_cast<const B*>(x), w_router, bias, T, d, renormalize, idx, gates, counts,
                                offsets, perm_token, perm_slot, slot_pos, gate_perm, static_cast<B*>(xp), status, s);
}

cudaError_t launch_combine(moe_dtype_t dtype, const float* y, int64_t split_stride, int32_t splits,
                           const int32_t* slot_pos, int64_t T, int64_t d, const void* residual,
                           const float* norm_weight, float norm_eps, void* out, uint32_t* status, cudaStream_t s) {
  if (residual || norm_weight) {
    if (dtype == MOE_F32)
      moe_combine_norm_kernel<float><<<static_cast<unsigned>(T), 256, 0, s>>>(
          y, split_stride, splits, slot_pos, d, static_cast<const float*>(residual), norm_weight, norm_eps,
          static_cast<float*>(out), status);
    else
      moe_combine_norm_kernel<__nv_bfloat16><<<static_cast<unsigned>(T), 256, 0, s>>>(
          y, split_stride, splits, slot_pos, d, static_cast<const __nv_bfloat16*>(residual), norm_weight,
          norm_eps, static_cast<__nv_bfloat16*>(out), status);
    return cudaGetLastError();
  }
  const int64_t n = T * (d / 4);
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(device_sm_count()) * 8);
  if (dtype == MOE_F32)
    moe_combine_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(y, split_stride, splits, slot_pos, T,
                                                                           d, static_cast<float*>(out), status);
  else
    moe_combine_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        y, split_stride, splits, slot_pos, T, d, static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Pieces of the expert-parallel form (experts split over GPUs, token rows
// exchanged between them); see moe_experts_forward and moe_gather_rows.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

// One CTA: counts of the n local experts into the kE slots the GEMM kernels
// schedule from (slots past n get no rows), their exclusive offsets, and 1.0
// into `ones` (gates of rows that carry none).
__global__ void moe_local_schedule_kernel(const int32_t* __restrict__ counts_in, int32_t n,
                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                          float* __restrict__ ones, int64_t n_ones) {
  if (threadIdx.x == 0) {
    int32_t off = 0;
    for (int e = 0; e < kE; ++e) {
      const int32_t c = e < n ? counts_in[e] : 0;
      counts[e] = c;
      offsets[e] = off;
      off += c;
    }
    offsets[kE] = off;
  }
  if (ones != nullptr)
    for (int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.x) * blockDim.x; i < n_ones;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
      ones[i] = 1.0f;
}

// y[i] = sum over s of part[s][i], s ascending from 0 (fixed order).
__global__ void __launch_bounds__(256) moe_sum_splits_kernel(const float* __restrict__ part, int64_t split_stride,
                                                             int32_t splits, int64_t n4, float* __restrict__ y) {
  for (int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.x) * blockDim.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
      const float4 v = reinterpret_cast<const float4*>(part + s * split_stride)[i];
      a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    reinterpret_cast<float4*>(y)[i] = a;
  }
}

// dst row i = src row index[i]; rows of `vecs` vectors of type V (16 or 4 bytes).
template <typename V>
__global__ void __launch_bounds__(256) moe_gather_rows_kernel(const V* __restrict__ src, int64_t src_rows,
                                                              const int32_t* __restrict__ index, int64_t n,
                                                              int64_t vecs, V* __restrict__ dst,
                                                              uint32_t* __restrict__ status) {
  const int64_t total = n * vecs;
  for (int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.x) * blockDim.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vecs, c = i - r * vecs;
    const int64_t from = index[r];
    if (kDebugBounds && !index_ok(from, src_rows)) {
      atomicOr(status, kStatusBounds);
      continue;
    }
    dst[i] = src[from * vecs + c];
  }
}

}  // namespace

cudaError_t launch_local_schedule(const int32_t* counts_in, int32_t n, int32_t* counts, int32_t* offsets,
                                  float* ones, int64_t n_ones, cudaStream_t s) {
  const int64_t blocks = ones ? std::min<int64_t>(std::max<int64_t>(1, (n_ones + 255) / 256), 1024) : 1;
  moe_local_schedule_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(counts_in, n, counts, offsets, ones,
                                                                          n_ones);
  return cudaGetLastError();
}

cudaError_t launch_sum_splits(const float* part, int64_t split_stride, int32_t splits, int64_t n, float* y,
                              cudaStream_t s) {
  const int64_t n4 = n / 4;
  const int64_t blocks = std::min<int64_t>(std::max<int64_t>(1, (n4 + 255) / 256), device_sm_count() * 8);
  moe_sum_splits_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(part, split_stride, splits, n4, y);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int64_t src_rows, const int32_t* index, int64_t n,
                               int64_t row_bytes, void* dst, uint32_t* status, cudaStream_t s) {
  // 16-byte vectors when the rows allow them, else 4-byte words.
  const bool wide = row_bytes % 16 == 0;
  const int64_t vecs = row_bytes / (wide ? 16 : 4);
  const int64_t blocks = std::min<int64_t>(std::max<int64_t>(1, (n * vecs + 255) / 256), device_sm_count() * 8);
  if (wide)
    moe_gather_rows_kernel<uint4><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const uint4*>(src), src_rows, index, n, vecs, static_cast<uint4*>(dst), status);
  else
    moe_gather_rows_kernel<uint32_t><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const uint32_t*>(src), src_rows, index, n, vecs, static_cast<uint32_t*>(dst), status);
  return cudaGetLastError();
}

}  // namespace moe
