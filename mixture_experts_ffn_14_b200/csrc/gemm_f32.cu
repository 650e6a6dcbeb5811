// gemm_f32.cu — fp32 grouped expert GEMMs on the CUDA cores (MOE_F32).
//
// Same operation as the tensor-core path (Grok-1 book ch. 10, section 10.4:
// down(GELU(x.Wg) * (x.Wu)) per expert) with true fp32 inputs and fp32
// accumulation: there is no fp32 tensor-core MMA (tf32 keeps 10 mantissa bits),
// so the fp32 form runs as shared-memory-tiled SIMT GEMMs. Tiles: 64 rows x 64
// columns, 256 threads, 4x4 outputs per thread, K in steps of 16; rows are the
// expert-contiguous permuted rows, tiles are enumerated on the device from the
// per-expert counts.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

struct F32Sched {
  int cnt[kE], off[kE], mt[kE], pre[kE + 1];
};

__device__ __forceinline__ void load_sched(F32Sched& s, const int32_t* counts, const int32_t* offsets, int nt,
                                           int64_t rows_total, uint32_t* status) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < kE; ++e) {
      s.cnt[e] = counts[e];
      s.off[e] = offsets[e];
      s.mt[e] = (s.cnt[e] + TM - 1) / TM;
      s.pre[e] = acc;
      acc += s.mt[e] * nt;
    }
    s.pre[kE] = acc;
    if (kDebugBounds && !expert_blocks_ok(counts, offsets, kE, rows_total)) {
      atomicOr(status, kStatusBounds);
      s.pre[kE] = 0;  // no tile: nothing is read or written through these rows
    }
  }
  __syncthreads();
}

__device__ __forceinline__ float act_ref(float z, int mode) {
  if (mode == MOE_ACT_GELU_ERF) return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
  if (mode == MOE_ACT_SILU) return z / (1.0f + expf(-z));
  return 0.5f * z * (1.0f + tanhf(0.7978845608028654f * (z + 0.044715f * z * z * z)));
}

// DUAL = true: acc0 = X.B0, acc1 = X.B1, out = act(acc0) * acc1    (gate/up)
// DUAL = false: out = rowscale[r] * X.B0                            (down)
template <bool DUAL>
__global__ void __launch_bounds__(256) moe_f32_expert_gemm(const float* __restrict__ X, const float* __restrict__ B0,
                                                           const float* __restrict__ B1,
                                                           const int32_t* __restrict__ counts,
                                                           const int32_t* __restrict__ offsets,
                                                           const float* __restrict__ rowscale, int K, int N,
                                                           int act, float* __restrict__ out, int64_t rows_total,
                                                           uint32_t* __restrict__ status) {
  __shared__ F32Sched sched;
  __shared__ float As[TK][TM];
  __shared__ float Bs0[TK][TN];
  __shared__ float Bs1[DUAL ? TK : 1][DUAL ? TN : 1];
  const int nt = N / TN;
  load_sched(sched, counts, offsets, nt, rows_total, status);
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;

  for (int tile = blockIdx.x; tile < sched.pre[kE]; tile += gridDim.x) {
    int e = 0;
    while (tile >= sched.pre[e + 1]) ++e;
    const int local = tile - sched.pre[e];
    const int mt = local % sched.mt[e];
    const int n0 = (local / sched.mt[e]) * TN;
    const int rows = min(TM, sched.cnt[e] - mt * TM);
    const int64_t row0 = sched.off[e] + static_cast<int64_t>(mt) * TM;
    const float* b0 = B0 + static_cast<int64_t>(e) * K * N;
    const float* b1 = DUAL ? B1 + static_cast<int64_t>(e) * K * N : nullptr;

    float acc0[4][4], acc1[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.0f;

    for (int k0 = 0; k0 < K; k0 += TK) {
      // A chunk [64 rows x 16 k], stored transposed.
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int li = tid + 256 * i;  // 0..1023
        const int r = li / TK, kk = li % TK;
        As[kk][r] = r < rows ? X[(row0 + r) * K + k0 + kk] : 0.0f;
      }
      {
        const int kk = tid / 16, c = (tid % 16) * 4;
        const float4 v0 = *reinterpret_cast<const float4*>(b0 + static_cast<int64_t>(k0 + kk) * N + n0 + c);
        Bs0[kk][c] = v0.x; Bs0[kk][c + 1] = v0.y; Bs0[kk][c + 2] = v0.z; Bs0[kk][c + 3] = v0.w;
        if (DUAL) {
          const float4 v1 = *reinterpret_cast<const float4*>(b1 + static_cast<int64_t>(k0 + kk) * N + n0 + c);
          Bs1[kk][c] = v1.x; Bs1[kk][c + 1] = v1.y; Bs1[kk][c + 2] = v1.z; Bs1[kk][c + 3] = v1.w;
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < TK; ++kk) {
        float a[4], p[4], q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          p[j] = Bs0[kk][tx * 4 + j];
          if (DUAL) q[j] = Bs1[kk][tx * 4 + j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc0[i][j] = fmaf(a[i], p[j], acc0[i][j]);
            if (DUAL) acc1[i][j] = fmaf(a[i], q[j], acc1[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      if (r >= rows) continue;
      const int64_t row = row0 + r;
      float o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        o[j] = DUAL ? act_ref(acc0[i][j], act) * acc1[i][j] : acc0[i][j] * rowscale[row];
      *reinterpret_cast<float4*>(out + row * N + n0 + tx * 4) = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

int f32_grid(int64_t T, int64_t N) {
  const int64_t tiles = ((2 * T) / TM + kE) * (N / TN);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, static_cast<int64_t>(device_sm_count()) * 4)));
}

}  // namespace

cudaError_t launch_f32_gateup(const float* xp, const float* wg, const float* wu, const int32_t* counts,
                              const int32_t* offsets, int64_t T, int64_t d, int64_t f, int32_t act,
                              float* h, uint32_t* status, cudaStream_t s) {
  moe_f32_expert_gemm<true><<<f32_grid(T, f), 256, 0, s>>>(xp, wg, wu, counts, offsets, nullptr,
                                                          static_cast<int>(d), static_cast<int>(f), act, h, 2 * T,
                                                          status);
  return cudaGetLastError();
}

cudaError_t launch_f32_down(const float* h, const float* wd, const int32_t* counts, const int32_t* offsets,
                            const float* gate_perm, int64_t T, int64_t d, int64_t f, float* y, uint32_t* status,
                            cudaStream_t s) {
  moe_f32_expert_gemm<false><<<f32_grid(T, d), 256, 0, s>>>(h, wd, nullptr, counts, offsets, gate_perm,
                                                           static_cast<int>(f), static_cast<int>(d), 0, y, 2 * T,
                                                           status);
  return cudaGetLastError();
}

}  // namespace moe
