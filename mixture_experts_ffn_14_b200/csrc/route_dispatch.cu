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

namespace moe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kTokPerWarp = kRouteTokens / (kRouterThreads / 32);  // 4

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
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
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
};

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

// One CTA = 32 tokens, one warp = 4 tokens; lanes split the hidden dimension in
// 16-byte vectors. Writes idx/gates per token and the CTA's per-expert slot count.
template <typename TX>
__global__ void __launch_bounds__(kRouterThreads) moe_router_kernel(const TX* __restrict__ x,
                                                                     const float* __restrict__ wr,
                                                                     const float* __restrict__ bias, int64_t T,
                                                                     int64_t d, int32_t renormalize,
                                                                     int32_t* __restrict__ idx,
                                                                     float* __restrict__ gates,
                                                                     int32_t* __restrict__ hist) {
  constexpr int V = Vec<TX>::N;
  __shared__ int cnt[kE];
  if (threadIdx.x < kE) cnt[threadIdx.x] = 0;
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokens + warp * kTokPerWarp;
  float acc[kTokPerWarp][kE];
#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[j][e] = 0.0f;

  for (int64_t c = static_cast<int64_t>(lane) * V; c < d; c += 32 * V) {
    float w[V][kE];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float4 a = *reinterpret_cast<const float4*>(wr + (c + i) * kE);
      const float4 b = *reinterpret_cast<const float4*>(wr + (c + i) * kE + 4);
      w[i][0] = a.x; w[i][1] = a.y; w[i][2] = a.z; w[i][3] = a.w;
      w[i][4] = b.x; w[i][5] = b.y; w[i][6] = b.z; w[i][7] = b.w;
    }
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j) {
      if (t0 + j < T) {
        float xv[V];
        Vec<TX>::load(x + (t0 + j) * d + c, xv);
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
          for (int e = 0; e < kE; ++e) acc[j][e] = fmaf(xv[i], w[i][e], acc[j][e]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[j][e] = warp_sum(acc[j][e]);

#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j) {
    const int64_t t = t0 + j;
    if (lane == j && t < T) {
      float l[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) l[e] = acc[j][e] + (bias ? bias[e] : 0.0f);
      // Top-2 by value; strict comparisons keep the lower index on ties.
      int e0 = 0;
#pragma unroll
      for (int e = 1; e < kE; ++e)
        if (l[e] > l[e0]) e0 = e;
      int e1 = e0 == 0 ? 1 : 0;
#pragma unroll
      for (int e = 0; e < kE; ++e)
        if (e != e0 && l[e] > l[e1]) e1 = e;
      const float m = l[e0];
      float s = 0.0f;
#pragma unroll
      for (int e = 0; e < kE; ++e) s += expf(l[e] - m);
      idx[2 * t] = e0;
      idx[2 * t + 1] = e1;
      const float p1 = expf(l[e1] - m);
      if (renormalize) {  // Mixtral: the two probabilities divided by their sum
        gates[2 * t] = 1.0f / (1.0f + p1);
        gates[2 * t + 1] = p1 / (1.0f + p1);
      } else {
        gates[2 * t] = 1.0f / s;
        gates[2 * t + 1] = p1 / s;
      }
      atomicAdd(&cnt[e0], 1);
      atomicAdd(&cnt[e1], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < kE) hist[static_cast<int64_t>(blockIdx.x) * kE + threadIdx.x] = cnt[threadIdx.x];
}

// Same 32-token range per CTA as the router. Each CTA sums the per-CTA
// histograms to find where its tokens land (no cross-CTA waiting), ranks its
// tokens per expert with warp ballots (token order = stable), writes the
// permutation arrays and copies the x rows to their permuted positions.
template <typename TX>
__global__ void __launch_bounds__(256) moe_dispatch_kernel(
    const TX* __restrict__ x, int64_t T, int64_t d, int64_t nblk, const int32_t* __restrict__ idx,
    const float* __restrict__ gates, const int32_t* __restrict__ hist, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token, int32_t* __restrict__ perm_slot,
    int32_t* __restrict__ slot_pos, float* __restrict__ gate_perm, TX* __restrict__ xp) {
  __shared__ int red[8][2 * kE];
  __shared__ int base[kE];
  __shared__ int pos_sm[kRouteTokens][2];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t blk = blockIdx.x;

  int tot[kE], pre[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) tot[e] = pre[e] = 0;
  for (int64_t c = threadIdx.x; c < nblk; c += blockDim.x) {
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const int v = hist[c * kE + e];
      tot[e] += v;
      if (c < blk) pre[e] += v;
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
      if (blk == 0) {
        counts[e] = total[e];
        offsets[e] = off;
      }
      off += total[e];
    }
    if (blk == 0) offsets[kE] = off;
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
    if (valid) {
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

  // Gather: 64 rows of d elements, as 16-byte vectors.
  const int64_t vec_per_row = d * static_cast<int64_t>(sizeof(TX)) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(xp);
  for (int64_t i = threadIdx.x; i < 2 * kRouteTokens * vec_per_row; i += blockDim.x) {
    const int r = static_cast<int>(i / vec_per_row);
    const int64_t c = i - r * vec_per_row;
    const int tl = r >> 1, s = r & 1;
    const int pos = pos_sm[tl][s];
    if (pos >= 0) dst[static_cast<int64_t>(pos) * vec_per_row + c] = src[(blk * kRouteTokens + tl) * vec_per_row + c];
  }
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
                                                          int64_t T, int64_t d, TO* __restrict__ out) {
  const int64_t q = d / 4;
  const int64_t n = T * q;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / q;
    const int64_t c = (i - t * q) * 4;
    const int64_t p0 = slot_pos[2 * t], p1 = slot_pos[2 * t + 1];
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int s = 0; s < splits; ++s) {
      const float4 u = *reinterpret_cast<const float4*>(y + s * split_stride + p0 * d + c);
      const float4 v = *reinterpret_cast<const float4*>(y + s * split_stride + p1 * d + c);
      a.x += u.x; a.y += u.y; a.z += u.z; a.w += u.w;
      b.x += v.x; b.y += v.y; b.z += v.z; b.w += v.w;
    }
    store4<TO>(out + t * d + c, make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w));
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
                                                               TO* __restrict__ out) {
  __shared__ float red[8];
  const int64_t t = blockIdx.x;
  const int64_t p0 = slot_pos[2 * t], p1 = slot_pos[2 * t + 1];
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

cudaError_t launch_router(moe_dtype_t dtype, const void* x, const float* w_router, const float* bias, int64_t T,
                          int64_t d, int32_t renormalize, int32_t* idx, float* gates, int32_t* hist,
                          cudaStream_t s) {
  const int64_t nblk = (T + kRouteTokens - 1) / kRouteTokens;
  if (dtype == MOE_F32)
    moe_router_kernel<float><<<static_cast<unsigned>(nblk), kRouterThreads, 0, s>>>(
        static_cast<const float*>(x), w_router, bias, T, d, renormalize, idx, gates, hist);
  else
    moe_router_kernel<__nv_bfloat16><<<static_cast<unsigned>(nblk), kRouterThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), w_router, bias, T, d, renormalize, idx, gates, hist);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(moe_dtype_t dtype, const void* x, int64_t T, int64_t d, int64_t nblk,
                            const int32_t* idx, const float* gates, const int32_t* hist, int32_t* counts,
                            int32_t* offsets, int32_t* perm_token, int32_t* perm_slot, int32_t* slot_pos,
                            float* gate_perm, void* xp, cudaStream_t s) {
  if (dtype == MOE_F32)
    moe_dispatch_kernel<float><<<static_cast<unsigned>(nblk), 256, 0, s>>>(
        static_cast<const float*>(x), T, d, nblk, idx, gates, hist, counts, offsets, perm_token, perm_slot,
        slot_pos, gate_perm, static_cast<float*>(xp));
  else
    moe_dispatch_kernel<__nv_bfloat16><<<static_cast<unsigned>(nblk), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), T, d, nblk, idx, gates, hist, counts, offsets, perm_token,
        perm_slot, slot_pos, gate_perm, static_cast<__nv_bfloat16*>(xp));
  return cudaGetLastError();
}

cudaError_t launch_combine(moe_dtype_t dtype, const float* y, int64_t split_stride, int32_t splits,
                           const int32_t* slot_pos, int64_t T, int64_t d, const void* residual,
                           const float* norm_weight, float norm_eps, void* out, cudaStream_t s) {
  if (residual || norm_weight) {
    if (dtype == MOE_F32)
      moe_combine_norm_kernel<float><<<static_cast<unsigned>(T), 256, 0, s>>>(
          y, split_stride, splits, slot_pos, d, static_cast<const float*>(residual), norm_weight, norm_eps,
          static_cast<float*>(out));
    else
      moe_combine_norm_kernel<__nv_bfloat16><<<static_cast<unsigned>(T), 256, 0, s>>>(
          y, split_stride, splits, slot_pos, d, static_cast<const __nv_bfloat16*>(residual), norm_weight,
          norm_eps, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
  }
  const int64_t n = T * (d / 4);
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(device_sm_count()) * 8);
  if (dtype == MOE_F32)
    moe_combine_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(y, split_stride, splits, slot_pos, T,
                                                                           d, static_cast<float*>(out));
  else
    moe_combine_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        y, split_stride, splits, slot_pos, T, d, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace moe
