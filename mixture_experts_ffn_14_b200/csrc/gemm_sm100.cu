// gemm_sm100.cu — grouped expert GEMMs on the 5th-generation tensor cores.
//
// Two kernels share one persistent, warp-specialised pipeline:
//   GATEUP: H[r, n] = act(Xp[r,:] . Wg[e][:, n]) * (Xp[r,:] . Wu[e][:, n])     (bf16 out)
//   DOWN:   Y[s, r, n] = gate[r] * (H[r, kslice_s] . Wd[e][kslice_s, n])         (fp32 out)
// for every permuted row r of expert e (rows are expert-contiguous after the
// dispatch stage). This is the GeGLU expert of the Grok-1 MoE sublayer (Grok-1
// book ch. 10, section 10.4, "GeGLU vs SwiGLU" box: down(act(up_1 x) * up_2 x)).
//
// Roles per CTA (one CTA per SM, persistent over a static tile list):
//   warp 0      TMA producer: activation tile + weight tile per 64-deep K stage
//   warp 1      TMEM allocator and tcgen05.mma issuer (one thread)
//   warps 4..7  epilogue: tcgen05.ld from TMEM, activation / gate / scale, global stores
//   warps 8..15 (int8 weights only) convert the int8 stage to fp16 in shared memory
//               (two warps per SM sub-partition, so one hides the other's latency)
//
// Shared memory per stage: X tile [128 rows x 64 K] bf16, K-major, 128-B swizzle
// (16 KB) and W tile = four chunks [64 K x 64 N] bf16, N(MN)-major, 128-B swizzle
// (32 KB); weights are used in the caller's [E, K, N] layout without a repack.
// int8 weights: the same tiles in fp16 (activations converted by the dispatch
// stage, weights by the converter warps), with the int8 staging in the TMA ring
// and the converted W tiles in a ring of their own (see Cfg).
//
// Orientation:
//   TOKEN_TILE    MMA M = 128 token rows (A = X, K-major), N = 256 weight columns
//                 (B = W, MN-major); one MMA per 16-deep K step.
//   WEIGHT_STREAM MMA M = 128 weight columns (A = W, MN-major), N = tokens of the
//                 tile rounded up to 16 (B = X, K-major); two MMAs per K step.
//                 Used when experts hold few tokens: every weight byte is read
//                 once, the down projection is split along K for parallelism.
// TMEM: 512 columns = two accumulator buffers of 256 columns, so the epilogue of
// one tile overlaps the main loop of the next.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "gemm_common.cuh"

namespace moe {
namespace tc {

constexpr int W_BYTES = 4 * WCHUNK;     // 32 KB: four [64 K x 64 N] chunks
constexpr int W8_BYTES = BK * 256;      // 16 KB int8 staging: two [64 K x 128 N] boxes
constexpr int XBOX_ROWS_WS = 32;        // WEIGHT_STREAM activation box height

// Shared memory. bf16 weights: STAGES slots of [X tile | W tile] (48 KB).
// int8 weights: two rings, so that more of the shared memory holds loads in
// flight: STAGES slots of [X tile | int8 W staging] (32 KB) filled by TMA, and
// CSTAGES slots of converted fp16 W tiles (32 KB) that the converter warps fill
// up to two stages ahead of the MMA (4 + 3 measured ~3 % faster than 5 + 2).
// TALL (int8 weights, token tiles): one tile covers 256 token rows; each
// converted W tile serves two M = 128 MMAs (rows 0-127 into accumulator
// columns 0-255, rows 128-255 into 256-511), so the conversion and the converted
// tile's shared-memory traffic per FLOP halve. The two halves of TMEM then hold
// one tile, and the epilogue no longer overlaps the next tile's main loop.
// SHORT (weight-stream tiles of at most 64 tokens, for small batches): the
// activation box of a slot shrinks to 8 KB, so the ring holds more weight
// stages in flight (int8: 6 slots = 96 KB of int8 weights instead of 4 = 64 KB;
// bf16: 5 slots = 160 KB instead of 128 KB). A weight-stream kernel streams
// every weight byte once with little reuse, so the bytes in flight per SM set
// its bandwidth.
template <bool W8, bool TALL = false, bool SHORT = false>
struct Cfg {
  static constexpr int XS_BYTES = SHORT ? 64 * 128 : (TALL ? 2 : 1) * X_BYTES;
  static constexpr int STAGES = SHORT ? (W8 ? 6 : 5) : (TALL ? 3 : 4);
  static constexpr int SLOT_BYTES = XS_BYTES + (W8 ? W8_BYTES : W_BYTES);
  static constexpr int CSTAGES = W8 ? ((TALL || SHORT) ? 2 : 3) : 0;
  static constexpr int RING_BYTES = STAGES * SLOT_BYTES + CSTAGES * W_BYTES;
  static constexpr int CONVERT_THREADS = 256;
  static constexpr int CONVERT_WARPS = CONVERT_THREADS / 32;
  // 256-row tiles: a second set of four epilogue warps (warps 8-11) takes rows
  // 128-255 while warps 4-7 take rows 0-127, halving the epilogue that these
  // tiles cannot overlap with the next tile's main loop. bf16 gate/up, median
  // of four alternating runs: T = 4096 5.685 -> 5.600 ms, T = 1024 1.711 ->
  // 1.703. int8 (640 threads, converters in warps 12-19; median of three
  // alternating runs): step T = 1024 2.959 -> 2.880 ms, T = 4096 9.587 -> 9.265.
  // bf16 256-row tiles run 16 epilogue warps (640 threads): each set of four
  // takes one 128-row half and one 64-column half of H (gate/up, median of
  // three alternating runs: T = 4096 5.468 -> 5.350 ms, T = 8192 10.53 -> 10.31).
  static constexpr int EPI_WARPS = TALL ? (W8 ? 8 : 16) : 4;
  static constexpr int THREADS = 128 + 32 * EPI_WARPS + (W8 ? CONVERT_THREADS : 0);
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM = RING_BYTES + BAR_BYTES + 1024;  // + alignment slack
};
constexpr int kMaxCStages = 4;  // barrier slots reserved for the converted-W ring
// Token tiles hand out their tiles in order from a global counter (zeroed by
// the caller) when one is given: the producer takes the next tile id when it
// starts a tile and passes it through a queue of kTileQS slots to the other
// roles (MMA thread, epilogue warps, converter warps), which read the tiles
// in the same order. A CTA that finishes early takes more tiles instead of
// idling (the tiles of one call differ in cost: short last row tiles, tall
// int8 tiles with one or two MMAs per step), and consecutive tile ids (the row
// tiles that share one weight tile) go to CTAs that became free together, so
// they read that weight tile from L2 close in time.
constexpr int kTileQS = 4;
// int8 weights: the converter warps form conv_groups(WS) groups that take the
// K-block steps in turn (group g converts steps n with n % groups == g), so
// that several steps are converted at once. Measured (two alternating runs
// each): weight-stream (decode, T = 64) 1.458 -> 1.420 ms with two groups;
// 256-row token tiles slower with two (T = 1024 2.91 -> 2.99 ms, T = 4096 8.94
// -> 9.16 ms), so they keep one group of eight warps on each step.
__host__ __device__ constexpr int conv_groups(bool ws) { return ws ? 2 : 1; }
static_assert(Cfg<true>::CSTAGES <= kMaxCStages && Cfg<true, true>::CSTAGES <= kMaxCStages &&
                  Cfg<true, false, true>::CSTAGES <= kMaxCStages,
              "converted-W ring deeper than its barrier slots");
static_assert((2 * Cfg<true, false, true>::STAGES + 2 * kMaxCStages + 4 + 2 * kTileQS) * 8 + 16 +
                      sizeof(SharedSched) + 4 * kTileQS <= Cfg<true>::BAR_BYTES,
              "barrier area too small");
static_assert(Cfg<true, true>::SMEM <= 232448 && Cfg<true>::SMEM <= 232448 && Cfg<false>::SMEM <= 232448 &&
                  Cfg<true, false, true>::SMEM <= 232448 && Cfg<false, false, true>::SMEM <= 232448,
              "shared memory above the per-block limit");

// TALL: 256-row token tiles (always with int8 weights; bf16 gate/up for
// larger batches, see launch_tc_gateup).
template <int KIND, bool WS, bool W8, bool SHORT = false, bool TALL = W8 && !WS>
__global__ void __launch_bounds__(Cfg<W8, TALL, SHORT>::THREADS, 1)
    moe_expert_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                           const __grid_constant__ CUtensorMap tm_w1, const Params p) {
  static_assert(!SHORT || WS, "short tiles are a weight-stream form");
  static_assert(!TALL || !WS, "tall tiles are a token-tile form");
  constexpr int TROWS = TALL ? 2 * BM : (SHORT ? BM / 2 : BM);  // token rows per tile
  constexpr int NACC = TALL ? 1 : 2;         // accumulator buffers in flight
  using C = Cfg<W8, TALL, SHORT>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-B swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* conv_area = smem + STAGES * C::SLOT_BYTES;  // int8: converted W ring
  uint8_t* bar_area = smem + C::RING_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);  // TMA slot filled
  uint64_t* empty_bar = full_bar + STAGES;                      // TMA slot free again
  uint64_t* cfull_bar = empty_bar + STAGES;                     // converted W slot ready
  uint64_t* cempty_bar = cfull_bar + kMaxCStages;               // converted W slot free again
  uint64_t* tfull_bar = cempty_bar + kMaxCStages;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* qfull_bar = tempty_bar + 2;        // tile-id queue slot written
  uint64_t* qempty_bar = qfull_bar + kTileQS;  // tile-id queue slot read by every consumer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty_bar + kTileQS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  SharedSched* sched = reinterpret_cast<SharedSched*>(tmem_slot + 4);
  volatile int* tile_q = reinterpret_cast<volatile int*>(sched + 1);

  if (skip_launch(p)) return;  // the other token-tile form takes this call

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      // int8: freed by the MMA commit (X read) and the converter warps of the
      // group that converted it (W8 read)
      mbar_init(&empty_bar[s], W8 ? 1 + C::CONVERT_WARPS / conv_groups(WS) : 1);
    }
    for (int c = 0; c < C::CSTAGES; ++c) {
      mbar_init(&cfull_bar[c], C::CONVERT_WARPS / conv_groups(WS));
      mbar_init(&cempty_bar[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 32 * C::EPI_WARPS);
    }
    for (int i = 0; i < kTileQS; ++i) {
      mbar_init(&qfull_bar[i], 1);
      // MMA thread, epilogue warps, converter warps
      mbar_init(&qempty_bar[i], 1 + C::EPI_WARPS + (W8 ? C::CONVERT_WARPS : 0));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w0);
    if (KIND == GATEUP) tma_prefetch_desc(&tm_w1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) build_sched(*sched, p, TROWS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ---- tile order (see kTileQS). Queue operations return the tile id, -1
  // when no tile is left, -2 when a wait timed out.
  const bool dyn = !WS && p.tile_counter != nullptr;
  const int ntiles = sched->pre[kE];
  auto q_fill = [&](int i) -> int {  // producer, lane 0
    const int slot = i % kTileQS;
    const uint32_t ph = (i / kTileQS) & 1;
    if (!mbar_wait(&qempty_bar[slot], ph ^ 1, kWaitLimitNs) || *abort_flag) return -2;
    const int t = atomicAdd(p.tile_counter, 1);
    const int tile = t < ntiles ? t : -1;
    tile_q[slot] = tile;
    mbar_arrive(&qfull_bar[slot]);
    return tile;
  };
  auto q_take = [&](int i) -> int {  // the MMA thread
    const int slot = i % kTileQS;
    const uint32_t ph = (i / kTileQS) & 1;
    if (!mbar_wait(&qfull_bar[slot], ph, kWaitLimitNs) || *abort_flag) return -2;
    const int tile = tile_q[slot];
    mbar_arrive(&qempty_bar[slot]);
    return tile;
  };
  auto q_take_warp = [&](int i) -> int {  // a whole epilogue or converter warp, one arrive
    const int slot = i % kTileQS;
    const uint32_t ph = (i / kTileQS) & 1;
    if (!warp_wait(&qfull_bar[slot], ph, abort_flag)) return -2;
    const int tile = tile_q[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&qempty_bar[slot]);
    return tile;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    // Lane 0 waits for a free stage, arms its full barrier and loads the weight
    // boxes (and the activation box of materialised rows). With the row gather
    // each of the 32 lanes also loads four token rows of A straight from x.
    // The two variants are compiled separately: the plain one is lane 0 alone
    // with no warp-synchronous step, so its refill latency stays minimal.
    // Weight-stream tiles read each weight byte once: mark it evict-first so
    // it does not push the reused activations out of L2.
    const uint64_t wpolicy = policy_evict_first();
    auto load_w = [&](void* dst, const CUtensorMap* map, uint64_t* bar, int n, int k, int e) {
      if (WS) tma_load_3d_hint(dst, map, bar, n, k, e, wpolicy);
      else tma_load_3d(dst, map, bar, n, k, e);
    };
    auto produce = [&](auto gather_tag) {
      constexpr bool G = decltype(gather_tag)::value;
      int stage = 0;
      uint32_t phase = 0;
      Tile t;
      for (int i = 0;; ++i) {
        int tile = blockIdx.x + i * gridDim.x;
        if (dyn) {
          if (!G || lane == 0) tile = q_fill(i);
          if (G) tile = __shfl_sync(0xffffffffu, tile, 0);
          if (tile == -2) {
            if (!G || lane == 0) {
              atomicOr(p.status, kStatusProducerTimeout);
              *abort_flag = 1;
            }
            return;
          }
        }
        if (tile < 0 || !decode_tile(*sched, p, tile, TROWS, t)) break;
        int32_t rtok[4] = {0, 0, 0, 0};
        if (G) gather_rows(p, t, t.row0 + 4 * lane, rtok);
        const int nbox_x = WS ? (t.rows + XBOX_ROWS_WS - 1) / XBOX_ROWS_WS : 1;
        // A 256-row tile of at most 128 rows (the last of an expert) loads only
        // the first activation box: its second MMA is skipped. Gate/up T = 512,
        // two runs: 1.162 / 1.162 ms against 1.181 / 1.181 with both boxes.
        const uint32_t xbytes =
            WS ? nbox_x * XBOX_ROWS_WS * BK * 2 : ((TALL && !G && t.rows <= BM) ? X_BYTES : C::XS_BYTES);
        const uint32_t wbytes = W8 ? W8_BYTES : W_BYTES;
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
          uint8_t* xs = smem + stage * C::SLOT_BYTES;
          uint8_t* ws = xs + C::XS_BYTES;  // bf16 W tile, or the int8 staging (W8)
          uint8_t* w8 = ws;
          const int k0 = (t.kb0 + kb) * BK;
          if (!G || lane == 0) {
            mbar_arrive_expect_tx(&full_bar[stage], xbytes + wbytes);
            if (WS) {
              for (int b = 0; b < nbox_x; ++b)
                tma_load_2d(xs + b * XBOX_ROWS_WS * 128, &tm_x, &full_bar[stage], k0, t.row0 + b * XBOX_ROWS_WS);
            } else if (!G) {
              tma_load_2d(xs, &tm_x, &full_bar[stage], k0, t.row0);
              if (TALL && t.rows > BM) tma_load_2d(xs + X_BYTES, &tm_x, &full_bar[stage], k0, t.row0 + BM);
            }
            if (W8) {
              if (KIND == GATEUP) {
                load_w(w8, &tm_w0, &full_bar[stage], t.n0, k0, t.e);
                load_w(w8 + W8_BYTES / 2, &tm_w1, &full_bar[stage], t.n0, k0, t.e);
              } else {
                load_w(w8, &tm_w0, &full_bar[stage], t.n0, k0, t.e);
                load_w(w8 + W8_BYTES / 2, &tm_w0, &full_bar[stage], t.n0 + 128, k0, t.e);
              }
            } else {
              if (KIND == GATEUP) {
                // chunks 0,1: gate columns n0..n0+127; chunks 2,3: up columns n0..n0+127
                load_w(ws + 0 * WCHUNK, &tm_w0, &full_bar[stage], t.n0, k0, t.e);
                load_w(ws + 1 * WCHUNK, &tm_w0, &full_bar[stage], t.n0 + 64, k0, t.e);
                load_w(ws + 2 * WCHUNK, &tm_w1, &full_bar[stage], t.n0, k0, t.e);
                load_w(ws + 3 * WCHUNK, &tm_w1, &full_bar[stage], t.n0 + 64, k0, t.e);
              } else {
                for (int j = 0; j < 4; ++j)
                  load_w(ws + j * WCHUNK, &tm_w0, &full_bar[stage], t.n0 + 64 * j, k0, t.e);
              }
            }
          }
          if (G) {
            __syncwarp();  // the barrier is armed before any lane's gather can complete on it
            // Lane l fills A rows 4l .. 4l+3 (512 B, 128-B swizzled like one tall box).
            tma_gather4(xs + lane * 512, &tm_x, &full_bar[stage], k0, rtok[0], rtok[1], rtok[2], rtok[3]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    };
    if (!WS && KIND == GATEUP && p.row_token != nullptr) {
      if constexpr (!WS && KIND == GATEUP && !W8) produce(std::true_type{});
    } else if (lane == 0) {
      produce(std::false_type{});
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int cstage = 0;       // int8: converted W ring
      uint32_t cphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      Tile t;
      for (int i = 0;; ++i) {
        const int tile = dyn ? q_take(i) : static_cast<int>(blockIdx.x + i * gridDim.x);
        if (tile == -2) {
          atomicOr(p.status, kStatusMmaTimeout);
          *abort_flag = 1;
          goto mma_done;
        }
        if (tile < 0 || !decode_tile(*sched, p, tile, TROWS, t)) break;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, kWaitLimitNs) || *abort_flag) {
          atomicOr(p.status, kStatusMmaTimeout);
          *abort_flag = 1;
          goto mma_done;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        const uint32_t ntok = WS ? ((t.rows + 15) / 16) * 16 : 0;
        // int8 weights are converted to fp16 (exact), and the activations they
        // meet are fp16 too: one operand type per MMA.
        const uint32_t idesc = W8 ? (WS ? idesc_f16_f32(128, ntok, 1, 0) : idesc_f16_f32(128, 256, 0, 1))
                                  : (WS ? idesc_bf16_f32(128, ntok, 1, 0) : idesc_bf16_f32(128, 256, 0, 1));
        for (int kb = 0; kb < p.kb_per_split; ++kb) {
          // int8: the converted W tile, then the X tile of the same K block (its
          // TMA slot completed before the converters could start on it).
          if ((W8 && !mbar_wait(&cfull_bar[cstage], cphase, kWaitLimitNs)) ||
              !mbar_wait(&full_bar[stage], phase, kWaitLimitNs) || *abort_flag) {
            atomicOr(p.status, kStatusMmaTimeout);
            *abort_flag = 1;
            goto mma_done;
          }
          tc_fence_after();
          const uint32_t xs = smem_u32(smem + stage * C::SLOT_BYTES);
          const uint32_t ws = W8 ? smem_u32(conv_area + cstage * W_BYTES) : xs + C::XS_BYTES;
          const bool second_half = TALL && t.rows > BM;  // rows 128..255 of a tall tile
#pragma unroll
          for (int k16 = 0; k16 < BK / 16; ++k16) {
            const uint32_t accum = (kb | k16) != 0;
            // X: K-major, 8-row groups 1024 B apart; a 16-deep K step is 32 B
            // inside the swizzled 128-B row.
            const uint64_t xdesc = smem_desc_sw128(xs + k16 * 32, 16, 1024);
            if (WS) {
              // W as A: MN-major, 64-column chunks 8 KB apart (LBO), 8-deep K
              // groups 1024 B apart (SBO); a 16-deep K step is 2048 B.
              const uint64_t a0 = smem_desc_sw128(ws + k16 * 2048, WCHUNK, 1024);
              const uint64_t a1 = smem_desc_sw128(ws + 2 * WCHUNK + k16 * 2048, WCHUNK, 1024);
              umma_bf16(d_tmem, a0, xdesc, idesc, accum);
              umma_bf16(d_tmem + 128, a1, xdesc, idesc, accum);
            } else {
              const uint64_t wdesc = smem_desc_sw128(ws + k16 * 2048, WCHUNK, 1024);
              umma_bf16(d_tmem, xdesc, wdesc, idesc, accum);
              if (second_half)
                umma_bf16(d_tmem + 256, smem_desc_sw128(xs + X_BYTES + k16 * 32, 16, 1024), wdesc, idesc, accum);
            }
          }
          umma_commit(&empty_bar[stage]);
          if (W8) {
            umma_commit(&cempty_bar[cstage]);
            if (++cstage == C::CSTAGES) {
              cstage = 0;
              cphase ^= 1;
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        umma_commit(&tfull_bar[acc]);
        if (++acc == NACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    mma_done:;
    }
  } else if (warp >= 4 && warp < 4 + C::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue --
    const int q = warp % 4;  // TMEM lanes 32q .. 32q+31
    // Tall tiles: warps 4-7 and 8-11 take rows 0-127 and 128-255; with 16
    // epilogue warps (bf16), warps 12-19 do the same for the second half of
    // the H columns, the first eight for the first half.
    const bool split = C::EPI_WARPS >= 8;
    const int set = (warp - 4) / 4;
    const bool upper = split && (set & 1) != 0;
    const int c_half = C::EPI_WARPS == 16 ? (set >> 1) : -1;
    const int c_begin = c_half < 0 ? 0 : 64 * c_half, c_end = c_half < 0 ? 128 : c_begin + 64;
    constexpr int ECW = (W8 || C::EPI_WARPS == 16) ? 16 : 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    Tile t;
    for (int i = 0;; ++i) {
      const int tile = dyn ? q_take_warp(i) : static_cast<int>(blockIdx.x + i * gridDim.x);
      if (tile == -2) {
        atomicOr(p.status, kStatusEpilogueTimeout);
        *abort_flag = 1;
        break;
      }
      if (tile < 0 || !decode_tile(*sched, p, tile, TROWS, t)) break;
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag)) {
        atomicOr(p.status, kStatusEpilogueTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * 256;
      if (!WS) {
        if (!upper)
          epilogue_token_rows<KIND, W8, ECW>(p, t, tbase, 32 * q + lane, t.row0, min(t.rows, BM), c_begin, c_end);
        if (TALL && t.rows > BM && (upper || !split))  // rows 128..255: accumulator columns 256..511
          epilogue_token_rows<KIND, W8, ECW>(p, t, tbase + 256, 32 * q + lane, t.row0 + BM, t.rows - BM, c_begin,
                                             c_end);
      } else {
        // Weight-stream: TMEM lane = output column, TMEM column = token.
        const int ntok = ((t.rows + 15) / 16) * 16;
        if (KIND == GATEUP) {
          uint16_t* hout = static_cast<uint16_t*>(p.out);  // bf16, or fp16 with int8 weights
          const int n = t.n0 + 32 * q + lane;
          float sg = 1.0f, su = 1.0f;
          if (W8) {
            sg = __bfloat162float(p.s0[static_cast<int64_t>(t.e) * p.N + n]);
            su = __bfloat162float(p.s1[static_cast<int64_t>(t.e) * p.N + n]);
          }
          uint32_t f16_bad = 0;  // int8 weights: an H value beyond the fp16 range
#pragma unroll 1
          for (int c = 0; c < ntok; c += 32) {
            uint32_t g[32], u[32];
            tmem_ld32x2(tbase + c, tbase + 128 + c, g, u);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c + j < t.rows) {
                const float h = act_f32(__uint_as_float(g[j]) * sg, p.act) * (__uint_as_float(u[j]) * su);
                const uint16_t hv =
                    W8 ? __half_as_ushort(__float2half_rn(h)) : __bfloat16_as_ushort(__float2bfloat16_rn(h));
                if (W8) f16_bad |= static_cast<uint32_t>((hv & 0x7C00u) == 0x7C00u);
                hout[static_cast<int64_t>(t.row0 + c + j) * p.N + n] = hv;
              }
            }
          }
          if (W8 && f16_bad) atomicOr(p.status, kStatusFp16Range);
        } else {
          float* yout = static_cast<float*>(p.out) + static_cast<int64_t>(t.kb0 / p.kb_per_split) * p.split_stride;
          const int n_a = t.n0 + 32 * q + lane;
          const int n_b = n_a + 128;
          float sa = 1.0f, sb = 1.0f;
          if (W8) {
            sa = __bfloat162float(p.s0[static_cast<int64_t>(t.e) * p.N + n_a]);
            sb = __bfloat162float(p.s0[static_cast<int64_t>(t.e) * p.N + n_b]);
          }
#pragma unroll 1
          for (int c = 0; c < ntok; c += 32) {
            uint32_t a[32], b[32];
            tmem_ld32x2(tbase + c, tbase + 128 + c, a, b);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c + j < t.rows) {
                const int64_t row = t.row0 + c + j;
                const float gate = p.gate_perm[row];
                yout[row * p.N + n_a] = __uint_as_float(a[j]) * sa * gate;
                yout[row * p.N + n_b] = __uint_as_float(b[j]) * sb * gate;
              }
            }
          }
          if (p.combine_count != nullptr) ws_combine_arrive(p, t, q, lane);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == NACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (W8 && warp >= 4 + C::EPI_WARPS) {
    // ----------------------------------------------- int8 -> fp16 convert --
    // Staging: two int8 boxes [64 K][128 N] (row = 128 B) in TMA slot `stage`.
    // Target: converted slot `cstage`, four fp16 chunks [64 K][64 N] with the
    // 128-B swizzle (16-B unit u of row k stored at unit u ^ (k % 8)).
    constexpr int GROUPS = conv_groups(WS);
    constexpr int GWARPS = C::CONVERT_WARPS / GROUPS;  // warps per group
    constexpr int GTHREADS = 32 * GWARPS;
    const int grp = (warp - 4 - C::EPI_WARPS) / GWARPS;
    const int ct = threadIdx.x - 128 - 32 * C::EPI_WARPS - grp * GTHREADS;  // 0 .. GTHREADS-1 within the group
    int n = 0;  // K-block step of this CTA, counted over all its tiles
    Tile t;
    for (int i = 0;; ++i) {
      const int tile = dyn ? q_take_warp(i) : static_cast<int>(blockIdx.x + i * gridDim.x);
      if (tile == -2) {
        atomicOr(p.status, kStatusConvertTimeout);
        *abort_flag = 1;
        goto convert_done;
      }
      if (tile < 0 || !decode_tile(*sched, p, tile, TROWS, t)) break;
      for (int kb = 0; kb < p.kb_per_split; ++kb, ++n) {
        if (n % GROUPS != grp) continue;  // another group's step
        const int stage = n % STAGES;
        const uint32_t phase = (n / STAGES) & 1;
        constexpr int CS = C::CSTAGES > 0 ? C::CSTAGES : 1;  // (this branch runs with int8 weights only)
        const int cstage = n % CS;
        const uint32_t cphase = (n / CS) & 1;
        if (!warp_wait(&full_bar[stage], phase, abort_flag) || !warp_wait(&cempty_bar[cstage], cphase ^ 1, abort_flag)) {
          atomicOr(p.status, kStatusConvertTimeout);
          *abort_flag = 1;
          goto convert_done;
        }
        {
          const uint8_t* w8 = smem + stage * C::SLOT_BYTES + C::XS_BYTES;
          uint8_t* wc = conv_area + cstage * W_BYTES;
#pragma unroll
          for (int it = 0; it < 1024 / GTHREADS; ++it) convert_int8_segment(w8, wc, ct + GTHREADS * it);
        }
        fence_proxy_async_smem();  // this thread's converted stores visible to the async proxy
        __syncwarp();              // ... and the whole warp's, before one arrive per warp
        if (lane == 0) {
          mbar_arrive(&empty_bar[stage]);  // staging slot read
          mbar_arrive(&cfull_bar[cstage]);
        }
      }
    }
  convert_done:;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int KIND, bool WS, bool W8, bool SHORT = false, bool TALL = W8 && !WS>
cudaError_t launch_one(const TcGemmArgs& a, cudaStream_t stream) {
  using C = Cfg<W8, TALL, SHORT>;
  auto kern = moe_expert_gemm_kernel<KIND, WS, W8, SHORT, TALL>;
  const cudaError_t err = set_smem_limit_once(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;

  CUtensorMap tm_x, tm_w0, tm_w1;
  {
    // Row gather: the map covers x itself and its box is one row high.
    const bool gather = !WS && KIND == GATEUP && a.row_token != nullptr;
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(gather ? a.x_rows : a.rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K) * 2};
    const uint32_t box[2] = {BK, static_cast<uint32_t>(gather ? 1 : WS ? XBOX_ROWS_WS : BM)};
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
  p.row_token = (!WS && KIND == GATEUP) ? a.row_token : nullptr;
  p.tile_counter = WS ? nullptr : a.tile_counter_single;  // token tiles: dynamic order when given
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
  p.group_rows = row_group_size(TALL ? 2 * BM : BM, int64_t(p.kb_per_split) * BK, kL2GroupBytes);
  p.group_limit = WS ? (1 << 30) : row_group_size(TALL ? 2 * BM : BM, int64_t(p.kb_per_split) * BK, kL2UngroupedBytes);
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

  // Upper bound of the tile count (the exact count is only known on device).
  const int64_t mtiles_max = a.rows / (TALL ? 2 * BM : (SHORT ? BM / 2 : BM)) + kE;
  const int64_t tiles_max = mtiles_max * (a.N / p.ntile) * p.splits;
  const int grid = static_cast<int>(std::min<int64_t>(tiles_max, device_sm_count()));
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(tm_x, tm_w0, tm_w1, p);
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_tc_gateup(const TcGemmArgs& a, cudaStream_t s) {
  if (a.weight_stream && a.short_tiles)
    return a.int8_weights ? tc::launch_one<tc::GATEUP, true, true, true>(a, s)
                          : tc::launch_one<tc::GATEUP, true, false, true>(a, s);
  if (a.weight_stream)
    return a.int8_weights ? tc::launch_one<tc::GATEUP, true, true>(a, s) : tc::launch_one<tc::GATEUP, true, false>(a, s);
  if (a.int8_weights) return tc::launch_one<tc::GATEUP, false, true>(a, s);
  // bf16 gate/up in 256-row tiles: each weight tile feeds two M = 128 MMAs on
  // one SM, which halves the weight bytes each SM reads from L2 per FLOP
  // (measured gate/up T = 1024 / 4096 / 8192: 1.71 / 5.64-5.68 / 11.0-11.5 ms
  // against 1.78 / 5.84-5.95 / 11.4-12.0 ms for the CTA-pair form).
  return a.tall_tiles ? tc::launch_one<tc::GATEUP, false, false, false, true>(a, s)
                      : tc::launch_one<tc::GATEUP, false, false>(a, s);
}

cudaError_t launch_tc_down(const TcGemmArgs& a, cudaStream_t s) {
  if (a.weight_stream && a.short_tiles)
    return a.int8_weights ? tc::launch_one<tc::DOWN, true, true, true>(a, s)
                          : tc::launch_one<tc::DOWN, true, false, true>(a, s);
  if (a.weight_stream)
    return a.int8_weights ? tc::launch_one<tc::DOWN, true, true>(a, s) : tc::launch_one<tc::DOWN, true, false>(a, s);
  return a.int8_weights ? tc::launch_one<tc::DOWN, false, true>(a, s) : tc::launch_one<tc::DOWN, false, false>(a, s);
}

}  // namespace moe
