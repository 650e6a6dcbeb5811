// gemm_sm100_pair.cu — token-tile grouped expert GEMMs on CTA pairs.
//
// Same operation as the single-CTA token-tile kernel (gemm_sm100.cu; the GeGLU
// expert of Grok-1 book ch. 10, section 10.4), computed by clusters of two CTAs
// on an SM pair with tcgen05.mma.cta_group::2: one MMA covers 256 token rows x
// 256 weight columns. Each CTA loads only its own half of the operands:
//   A (activations): this CTA's 128 token rows         [128 x 64 K], 16 KB/stage
//   B (weights):     this CTA's 128 of the 256 columns  [64 K x 128 N], 16 KB/stage
// and keeps its 128 rows of the accumulator in its own TMEM, so the epilogue
// is the single-CTA one. Per stage a CTA moves 32 KB instead of 48 KB for the
// same MMA work per SM, which leaves room for 6 stages in flight.
//
// Synchronisation (bf16 weights): the even CTA's producer expects the bytes
// of both CTAs on its own full barrier; both CTAs' TMA loads (cta_group::2
// form, no multicast) complete on it. The even CTA's single MMA thread issues
// the pair MMAs and releases a stage / hands over an accumulator with
// tcgen05.commit multicast to the barriers of both CTAs. Epilogue warps of
// both CTAs arrive on the even CTA's accumulator-empty barrier.
// int8 weights: each CTA's loads complete on its own full barrier; its
// converter warps turn its int8 half into fp16 and arrive on the even CTA's
// converted barrier, on which the MMA thread waits.
// Every wait is bounded; a timeout records a status bit and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "gemm_common.cuh"

namespace moe {
namespace tc {

constexpr int PAIR_ROWS = 2 * BM;      // 256 token rows per pair tile
constexpr int PW_BYTES = 2 * WCHUNK;   // 16 KB: this CTA's 128 weight columns
constexpr int PW8_BYTES = BK * 128;    // 8 KB: one int8 box [64 K x 128 N]

// Tile order. With bf16 weights the pair kernel hands out tiles dynamically:
// the even CTA's producer takes the next tile id from a global counter when it
// starts a tile, and writes it into slot i % kTileQ of both CTAs' tile-id
// queues; every other role reads its tiles from its own CTA's queue in the same
// order and frees the slot on the even CTA's qempty barrier. Consecutive tile
// ids are the row tiles that share one weight tile, and they go to the pairs that
// become free together, so those pairs read the weight tile from L2 close in
// time. (With static round-robin order the pairs that share a weight tile change
// every wave and drift apart, and the weights are fetched from DRAM again.)
// int8 weights keep the static order: their converter warps would be a third
// kind of reader.
constexpr int kTileQ = 4;            // producer leads the epilogue by at most 3 tiles
constexpr int kTileQConsumers = 10;  // odd producer, MMA thread, 4 epilogue warps x 2 CTAs

template <bool W8>
struct PairCfg {
  static constexpr int STAGES = W8 ? 5 : 6;
  static constexpr int STAGE_BYTES = X_BYTES + PW_BYTES + (W8 ? PW8_BYTES : 0);
  static constexpr int CONVERT_THREADS = 256;
  static constexpr int CONVERT_WARPS = CONVERT_THREADS / 32;
  static constexpr int THREADS = W8 ? 256 + CONVERT_THREADS : 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 1024;  // barriers + alignment slack
};

// Bounded wait with cluster-scope acquire (for barriers that other CTAs arrive on).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (try_once()) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

template <int KIND, bool W8>
__global__ void __launch_bounds__(PairCfg<W8>::THREADS, 1)
    moe_expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                                const __grid_constant__ CUtensorMap tm_w1, const Params p) {
  using C = PairCfg<W8>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bar_area = smem + STAGES * C::STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* conv_bar = empty_bar + STAGES;
  uint64_t* tfull_bar = conv_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* qfull_bar = tempty_bar + 2;      // tile-id queue slot written
  uint64_t* qempty_bar = qfull_bar + kTileQ;  // tile-id queue slot read by every role (even CTA's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty_bar + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  SharedSched* sched = reinterpret_cast<SharedSched*>(tmem_slot + 4);
  volatile int* tile_q = reinterpret_cast<volatile int*>(sched + 1);

  if (skip_launch(p)) return;  // the other token-tile form takes this call

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs of the pair
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&conv_bar[s], 2 * C::CONVERT_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 2 * 4);  // four epilogue warps in each CTA
    }
    for (int i = 0; i < kTileQ; ++i) {
      mbar_init(&qfull_bar[i], 1);
      mbar_init(&qempty_bar[i], kTileQConsumers);
    }
    *abort_flag = 0;
    build_sched(*sched, p, PAIR_ROWS);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w0);
    if (KIND == GATEUP) tma_prefetch_desc(&tm_w1);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ---- tile order (see kTileQ). Queue operations return the tile id, -1 when
  // no tile is left, -2 when a wait timed out.
  const bool dyn = !W8 && p.tile_counter != nullptr;
  const int ntiles = sched->pre[kE];
  auto q_fill = [&](int i) -> int {  // even CTA's producer
    const int slot = i % kTileQ;
    const uint32_t ph = (i / kTileQ) & 1;
    if (!mbar_wait_cluster(&qempty_bar[slot], ph ^ 1, kWaitLimitNs) || *abort_flag) return -2;
    const int t = atomicAdd(p.tile_counter, 1);
    const int tile = t < ntiles ? t : -1;
    tile_q[slot] = tile;
    st_shared_cluster_u32(mapa_shared(const_cast<int*>(&tile_q[slot]), 1), static_cast<uint32_t>(tile));
    mbar_arrive(&qfull_bar[slot]);
    mbar_arrive_cluster(mapa_shared(&qfull_bar[slot], 1));
    return tile;
  };
  auto q_take = [&](int i) -> int {  // one thread of any other role
    const int slot = i % kTileQ;
    const uint32_t ph = (i / kTileQ) & 1;
    if (!mbar_wait_cluster(&qfull_bar[slot], ph, kWaitLimitNs) || *abort_flag) return -2;
    const int tile = tile_q[slot];
    mbar_arrive_cluster(mapa_shared(&qempty_bar[slot], 0));
    return tile;
  };
  auto q_take_warp = [&](int i) -> int {  // a whole epilogue warp, one arrive
    const int slot = i % kTileQ;
    const uint32_t ph = (i / kTileQ) & 1;
    const bool ok = mbar_wait_cluster(&qfull_bar[slot], ph, kWaitLimitNs) && !*abort_flag;
    if (!__all_sync(0xffffffffu, ok)) return -2;
    const int tile = tile_q[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa_shared(&qempty_bar[slot], 0));
    return tile;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    // Lane 0 waits for a free stage, arms the barrier and loads the weight box
    // (and the activation box of materialised rows); with the row gather each
    // of the 32 lanes also loads four of this CTA's 128 token rows from x. The
    // two variants are compiled separately so that the plain one stays lane 0
    // alone with no warp-synchronous step.
    auto produce = [&](auto gather_tag) {
      constexpr bool G = decltype(gather_tag)::value;
      int stage = 0;
      uint32_t phase = 0;
      Tile t;
      for (int i = 0;; ++i) {
        int tile = pair + i * npairs;
        if (dyn) {
          if (!G || lane == 0) tile = rank == 0 ? q_fill(i) : q_take(i);
          if (G) tile = __shfl_sync(0xffffffffu, tile, 0);
          if (tile == -2) {
            if (!G || lane == 0) {
              atomicOr(p.status, kStatusProducerTimeout);
              *abort_flag = 1;
            }
            return;
          }
        }
        if (tile < 0 || !decode_tile(*sched, p, tile, PAIR_ROWS, t)) break;
        const int row = t.row0 + BM * static_cast<int>(rank);
        int32_t rtok[4] = {0, 0, 0, 0};
        if (G) gather_rows(p, t, row + 4 * lane, rtok);
        // GATEUP: the even CTA holds the gate columns, the odd one the up
        // columns (accumulator columns 0..127 / 128..255). DOWN: 128 columns each.
        const CUtensorMap* wmap = (KIND == GATEUP && rank == 1) ? &tm_w1 : &tm_w0;
        const int n = KIND == GATEUP ? t.n0 : t.n0 + 128 * static_cast<int>(rank);
        for (int kb = 0; kb < p.kb_per_split; ++kb) {
          int ok = 1;
          if (!G || lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, kWaitLimitNs) && !*abort_flag;
          if (G) ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (!G || lane == 0) {
              atomicOr(p.status, kStatusProducerTimeout);
              *abort_flag = 1;
            }
            return;
          }
          uint8_t* xs = smem + stage * C::STAGE_BYTES;
          uint8_t* ws = xs + X_BYTES;
          uint8_t* w8 = ws + PW_BYTES;
          const int k0 = (t.kb0 + kb) * BK;
          if (W8) {
            if (!G || lane == 0) {
              mbar_arrive_expect_tx(&full_bar[stage], X_BYTES + PW8_BYTES);
              if (!G) tma_load_2d(xs, &tm_x, &full_bar[stage], k0, row);
              tma_load_3d(w8, wmap, &full_bar[stage], n, k0, t.e);
            }
            if (G) {
              __syncwarp();  // armed before any lane's gather can complete on it
              tma_gather4(xs + lane * 512, &tm_x, &full_bar[stage], k0, rtok[0], rtok[1], rtok[2], rtok[3]);
            }
          } else {
            const uint32_t bar0 = mapa_shared(&full_bar[stage], 0);
            if (!G || lane == 0) {
              if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * (X_BYTES + PW_BYTES));
              if (!G) tma_load_2d_pair(xs, &tm_x, bar0, k0, row);
              tma_load_3d_pair(ws, wmap, bar0, n, k0, t.e);
              tma_load_3d_pair(ws + WCHUNK, wmap, bar0, n + 64, k0, t.e);
            }
            if (G) {
              __syncwarp();
              tma_gather4_pair(xs + lane * 512, &tm_x, bar0, k0, rtok[0], rtok[1], rtok[2], rtok[3]);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: every stage's last release (an arrive sent by the pair's MMA
      // commit) has landed before this CTA may exit.
      if (!G || lane == 0) {
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, kWaitLimitNs)) {
            atomicOr(p.status, kStatusProducerTimeout);
            break;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    };
    if (KIND == GATEUP && p.row_token != nullptr) {
      if constexpr (KIND == GATEUP) produce(std::true_type{});
    } else if (lane == 0) {
      produce(std::false_type{});
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      // int8 weights: fp16 operands on both sides (exact conversion).
      const uint32_t idesc = W8 ? idesc_f16_f32(PAIR_ROWS, 256, 0, 1) : idesc_bf16_f32(PAIR_ROWS, 256, 0, 1);
      Tile t;
      for (int i = 0;; ++i) {
        const int tile = dyn ? q_take(i) : pair + i * npairs;
        if (tile == -2) {
          atomicOr(p.status, kStatusMmaTimeout);
          *abort_flag = 1;
          goto mma_done;
        }
        if (tile < 0 || !decode_tile(*sched, p, tile, PAIR_ROWS, t)) break;
        if (!mbar_wait_cluster(&tempty_bar[acc], acc_phase ^ 1, kWaitLimitNs) || *abort_flag) {
          atomicOr(p.status, kStatusMmaTimeout);
          *abort_flag = 1;
          goto mma_done;
        }
        tc_fence_after();
        {
          const uint32_t d_tmem = tmem_base + acc * 256;
          for (int kb = 0; kb < p.kb_per_split; ++kb) {
            const bool ok = W8 ? mbar_wait_cluster(&conv_bar[stage], phase, kWaitLimitNs)
                               : mbar_wait(&full_bar[stage], phase, kWaitLimitNs);
            if (!ok || *abort_flag) {
              atomicOr(p.status, kStatusMmaTimeout);
              *abort_flag = 1;
              goto mma_done;
            }
            tc_fence_after();
            const uint32_t xs = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t ws = xs + X_BYTES;
#pragma unroll
            for (int k16 = 0; k16 < BK / 16; ++k16) {
              const uint64_t adesc = smem_desc_sw128(xs + k16 * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(ws + k16 * 2048, WCHUNK, 1024);
              umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | k16) != 0);
            }
            umma_commit_pair(&empty_bar[stage], 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          umma_commit_pair(&tfull_bar[acc], 0x3);
        }
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    mma_done:;
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue --
    const int q = warp - 4;
    const uint32_t tempty0_a = mapa_shared(&tempty_bar[0], 0);
    const uint32_t tempty0_b = mapa_shared(&tempty_bar[1], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    Tile t;
    for (int i = 0;; ++i) {
      const int tile = dyn ? q_take_warp(i) : pair + i * npairs;
      if (tile == -2) {
        atomicOr(p.status, kStatusEpilogueTimeout);
        *abort_flag = 1;
        break;
      }
      if (tile < 0 || !decode_tile(*sched, p, tile, PAIR_ROWS, t)) break;
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag)) {
        atomicOr(p.status, kStatusEpilogueTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * 256;
      const int cta_rows = BM * static_cast<int>(rank);
      epilogue_token_rows<KIND, W8>(p, t, tbase, 32 * q + lane, t.row0 + cta_rows, t.rows - cta_rows);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty0_b : tempty0_a);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (W8 && warp >= 8) {
    // ----------------------------------------------- int8 -> fp16 convert --
    const int ct = threadIdx.x - 256;
    int stage = 0;
    uint32_t phase = 0;
    Tile t;
    for (int tile = pair; decode_tile(*sched, p, tile, PAIR_ROWS, t); tile += npairs) {
      for (int kb = 0; kb < p.kb_per_split; ++kb) {
        if (!warp_wait(&full_bar[stage], phase, abort_flag)) {
          atomicOr(p.status, kStatusConvertTimeout);
          *abort_flag = 1;
          goto convert_done;
        }
        {
          uint8_t* xs = smem + stage * C::STAGE_BYTES;
          uint8_t* ws = xs + X_BYTES;
          const uint8_t* w8 = ws + PW_BYTES;
#pragma unroll
          for (int it = 0; it < 512 / C::CONVERT_THREADS; ++it)
            convert_int8_segment(w8, ws, ct + C::CONVERT_THREADS * it);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(&conv_bar[stage], 0));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  convert_done:;
  }

  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <int KIND, bool W8>
cudaError_t launch_pair(const TcGemmArgs& a, cudaStream_t stream) {
  using C = PairCfg<W8>;
  auto kern = moe_expert_gemm_pair_kernel<KIND, W8>;
  const cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  // Clusters of two that fit at once on this device (queried once per device).
  const int max_pairs = once_per_device(reinterpret_cast<const void*>(&launch_pair<KIND, W8>), [](const void*) {
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
    c.blockDim = dim3(PairCfg<W8>::THREADS, 1, 1);
    c.dynamicSmemBytes = PairCfg<W8>::SMEM;
    c.attrs = &at;
    c.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, moe_expert_gemm_pair_kernel<KIND, W8>, &c) != cudaSuccess || n <= 0)
      n = device_sm_count() / 2;
    return n;
  });

  CUtensorMap tm_x, tm_w0, tm_w1;
  {
    // Row gather: the map covers x itself and its box is one row high.
    const bool gather = KIND == GATEUP && a.row_token != nullptr;
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(gather ? a.x_rows : a.rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K) * 2};
    const uint32_t box[2] = {BK, static_cast<uint32_t>(gather ? 1 : BM)};
    if (!encode_tensor_map(&tm_x, W8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.x,
                           dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K),
                              static_cast<uint64_t>(a.n_experts > 0 ? a.n_experts : kE)};
    const uint64_t esz = W8 ? 1 : 2;
    const uint64_t strides[2] = {static_cast<uint64_t>(a.N) * esz, static_cast<uint64_t>(a.N) * a.K * esz};
    const uint32_t box[3] = {static_cast<uint32_t>(W8 ? 128 : 64), BK, 1};
    const CUtensorMapDataType dt = W8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = W8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!encode_tensor_map(&tm_w0, dt, 3, a.w0, dims, strides, box, sw)) return cudaErrorInvalidValue;
    if (!encode_tensor_map(&tm_w1, dt, 3, KIND == GATEUP ? a.w1 : a.w0, dims, strides, box, sw))
      return cudaErrorInvalidValue;
  }

  Params p;
  p.counts = a.counts;
  p.offsets = a.offsets;
  p.gate_perm = a.gate_perm;
  p.row_token = KIND == GATEUP ? a.row_token : nullptr;
  p.tile_counter = W8 ? nullptr : a.tile_counter;
  p.s0 = a.s0;
  p.s1 = a.s1;
  p.out = a.out;
  p.rows = a.rows;
  p.split_stride = a.rows * static_cast<int64_t>(a.N);
  p.K = a.K;
  p.N = a.N;
  p.splits = KIND == DOWN ? a.splits : 1;
  p.kb_per_split = a.K / BK / p.splits;
  p.ntile = KIND == GATEUP ? 128 : 256;
  // L2 groups of row tiles (tile_order.cuh): experts whose activation rows
  // (this K split) exceed 96 MB go in groups of 64 MB.
  p.group_rows = row_group_size(PAIR_ROWS, int64_t(p.kb_per_split) * BK, kL2GroupBytes);
  p.group_limit = row_group_size(PAIR_ROWS, int64_t(p.kb_per_split) * BK, kL2UngroupedBytes);
  p.act = a.act;
  p.select = a.select;
  p.sm_count = device_sm_count();
  p.status = a.status;
  const bool fuse = KIND == DOWN && a.combine_count != nullptr;
  p.perm_token = fuse ? a.perm_token : nullptr;
  p.slot_pos = fuse ? a.slot_pos : nullptr;
  p.combine_count = fuse ? a.combine_count : nullptr;
  p.combine_out = fuse ? static_cast<__nv_bfloat16*>(a.combine_out) : nullptr;
  p.residual = fuse ? static_cast<const __nv_bfloat16*>(a.residual) : nullptr;

  const int64_t ptiles_max = (a.rows / PAIR_ROWS + kE) * (a.N / p.ntile) * p.splits;
  const int pairs = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ptiles_max, max_pairs)));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w0, tm_w1, p);
}

}  // namespace tc

cudaError_t launch_tc_gateup_pair(const TcGemmArgs& a, cudaStream_t s) {
  return a.int8_weights ? tc::launch_pair<tc::GATEUP, true>(a, s) : tc::launch_pair<tc::GATEUP, false>(a, s);
}

cudaError_t launch_tc_down_pair(const TcGemmArgs& a, cudaStream_t s) {
  return a.int8_weights ? tc::launch_pair<tc::DOWN, true>(a, s) : tc::launch_pair<tc::DOWN, false>(a, s);
}

}  // namespace moe
