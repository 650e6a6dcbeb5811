/*
 * moe.h — C ABI of the B200 (sm_100a) Grok-1 MoE feed-forward sublayer.
 *
 * The operation (grok-field-guide "Grok-1 blueprint", section "MoE sublayer";
 * Grok-1 book ch. 10 "Comparison with other MoE", sections 10.3, 10.3.1, 10.4):
 *   for every token t (row of x):
 *     logits = x[t] . w_router (+ router_bias)           fp32, 8 experts
 *     p      = softmax(logits)                           fp32
 *     (e0,e1)= the two largest logits, descending; an exact tie goes to the
 *              lower expert index; gates g0 = p[e0], g1 = p[e1], NOT renormalised
 *     y_s    = ( GELU(x[t] . w_gate[e_s]) * (x[t] . w_up[e_s]) ) . w_down[e_s]
 *     out[t] = g0 * y_0 + g1 * y_1
 *   GELU is the tanh approximation unless MOE_ACT_GELU_ERF is asked for. Every
 *   routed (token, expert) pair is computed: no capacity limit, no token drop
 *   (Grok-1 book ch. 10, section 10.3.2, capacity-factor box).
 * Options (moe_options_t) add the variants the same pages compare against:
 *   renormalize = 1: gates divided by g0 + g1 (Mixtral, ch. 10 section 10.3.1);
 *   MOE_ACT_SILU: SiLU instead of GELU on the gate branch (SwiGLU, section 10.4);
 *   post_norm_weight / residual: out[t] = residual[t] + w * y / sqrt(mean(y^2) + eps)
 *   with y the gate-weighted sum above, the sublayer's post-RMSNorm and residual
 *   add (sandwich norm, section 10.3.1; the blueprint's "added back to the trunk").
 *
 * Pointers. Every array argument is a DEVICE pointer on the device that owns
 * `stream`; the caller owns all of them; the library never frees or retains
 * them and never synchronises the stream. All arrays are dense, row-major,
 * 16-byte aligned:
 *   x        [T, d]      fp32 (MOE_F32) or bf16 (MOE_BF16, MOE_BF16_INT8W)
 *   w_router [d, E]      fp32 (always)
 *   w_gate   [E, d, f]   fp32 / bf16 / int8 (by dtype)
 *   w_up     [E, d, f]   fp32 / bf16 / int8
 *   w_down   [E, f, d]   fp32 / bf16 / int8
 *   out      [T, d]      same dtype as x
 * int8 weights carry one bf16 scale per output channel (Grok-1 book ch. 1,
 * section 1.2, INT8 box): w = q * s, s_gate/s_up [E, f], s_down [E, d].
 *
 * Limits of this version: E == 8, k == 2; MOE_F32 needs d % 64 == 0 and
 * f % 64 == 0; MOE_BF16 and MOE_BF16_INT8W need d % 256 == 0 and f % 128 == 0;
 * 0 <= T <= 2^24. T == 0 returns MOE_OK and launches nothing.
 *
 * Errors. Arguments are checked on the host before anything is launched; a
 * failed check returns its status and launches nothing. A launch failure
 * returns MOE_ERR_CUDA. Faults of earlier asynchronous work surface at the
 * caller's next synchronisation, not here. Kernels never trap: they record
 * what went wrong as bits of the workspace status word, which
 * moe_device_status() reads back as MOE_ERR_DEVICE_CHECK with the code:
 *   0x01, 0x02, 0x04, 0x08  a GEMM wait (producer, MMA, epilogue, int8
 *                           converter) exceeded its time limit; the kernel
 *                           unwound and the output is incomplete
 *   0x10                    moe_selftest_bounded_wait's wait ran out (expected)
 *   0x20                    MOE_BF16_INT8W: an activation or GeGLU intermediate
 *                           left the fp16 range (|v| > 65504 became infinite);
 *                           the output is not valid
 *   0x40                    library built with MOE_DEBUG_BOUNDS: an index
 *                           outside its array was caught and the access skipped
 * Behaviour on non-finite inputs is unspecified.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_EXPORT __attribute__((visibility("default")))
#else
#define MOE_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size   */
  MOE_ERR_UNSUPPORTED = 2,   /* E != 8, k != 2, or d / f not a supported multiple */
  MOE_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned              */
  MOE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than needed      */
  MOE_ERR_CUDA = 5,          /* a CUDA runtime / driver call failed           */
  MOE_ERR_DEVICE_CHECK = 6   /* a kernel recorded a device-side check failure */
} moe_status_t;

typedef enum {
  MOE_F32 = 0,         /* fp32 activations and weights, fp32 arithmetic        */
  MOE_BF16 = 1,        /* bf16 activations and weights, fp32 accumulation      */
  MOE_BF16_INT8W = 2   /* bf16 activations, int8 weights + bf16 channel scales;
                          the expert GEMMs run on fp16 operands: int8 -> fp16 is
                          exact, bf16 activations -> fp16 is exact for normal
                          values below 65504 in magnitude, and the GeGLU
                          intermediate is kept in fp16 (range |h| < 65504)     */
} moe_dtype_t;

/* Activation on the gate branch of every expert. */
typedef enum {
  MOE_ACT_GELU_TANH = 0,  /* GELU, tanh approximation (default, Grok-1) */
  MOE_ACT_GELU_ERF = 1,   /* GELU, z * Phi(z)                           */
  MOE_ACT_SILU = 2        /* SiLU, z * sigmoid(z) (Mixtral)             */
} moe_activation_t;

/* Kernel family. AUTO picks WEIGHT_STREAM (tokens on the MMA N side, split-K
 * down projection) when the average tokens per expert is small (T <= 128 with
 * bf16 weights, T <= 256 with int8 weights; measured crossovers), else token
 * tiles (tokens on the MMA M side). For those small bf16 batches only the down
 * projection streams its weights that way; the gate/up GEMM runs 128-token
 * tiles on single CTAs (measured faster). Above them, with bf16 weights the gate/up
 * GEMM then runs 256-token tiles on single CTAs from T = 512 on; below that,
 * and for the down GEMM, the device chooses from the expert counts between
 * 128-token tiles on single CTAs and 256-token tiles on CTA pairs
 * (cta_group::2). int8 weights take 256-token tiles on single CTAs.
 * TOKEN_TILE forces the pair form, TOKEN_TILE_SINGLE the single-CTA form
 * (128-token tiles for bf16). All compute the same result within rounding;
 * each H element accumulates the same K steps in the same order in every
 * token-tile form. */
typedef enum {
  MOE_PATH_AUTO = 0,
  MOE_PATH_TOKEN_TILE = 1,
  MOE_PATH_WEIGHT_STREAM = 2,
  MOE_PATH_TOKEN_TILE_SINGLE = 3
} moe_path_t;

/* Per-output-channel scales of int8 weights (device pointers, bf16). */
typedef struct {
  const void* s_gate; /* [E, f] */
  const void* s_up;   /* [E, f] */
  const void* s_down; /* [E, d] */
} moe_scales_t;

/* cudaStream_t, passed as an opaque handle (NULL = the legacy default stream). */
typedef void* moe_stream_t;

/* All arguments of one forward call (see the file header for layouts). */
typedef struct {
  const void* x;
  const float* w_router;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const moe_scales_t* w_scales; /* host struct of device pointers; NULL unless MOE_BF16_INT8W */
  void* out;
  int64_t T, d, f;
  int32_t E, k;
  moe_dtype_t dtype;
} moe_args_t;

/* Per-call options; a zero-initialised struct (or opts == NULL) is the plain
 * Grok-1 sublayer with automatic kernel choices. */
typedef struct {
  moe_activation_t activation; /* gate-branch activation, MOE_ACT_GELU_TANH default      */
  const float* router_bias;    /* [E] fp32 device pointer added to the logits, or NULL    */
  moe_path_t path;             /* kernel family; MOE_PATH_AUTO by default                */
  int32_t down_splits;         /* split-K factor for w_down (must divide f/64); 0 = auto  */
  void* const* stage_events;   /* NULL, or 6 cudaEvent_t (host array) recorded on the
                                  stream before router, dispatch, gate/up GEMM, down
                                  GEMM, combine, and after combine (stage timing)        */
  int32_t renormalize;         /* 0: gates are the softmax probabilities (Grok-1);
                                  1: gates divided by their sum (Mixtral)                */
  const void* residual;        /* [T, d] x-dtype device pointer added to the output, or NULL */
  const float* post_norm_weight; /* [d] fp32 RMSNorm weight applied to the sublayer
                                  output before the residual add, or NULL (no norm)      */
  float norm_eps;              /* RMSNorm epsilon (> 0) when post_norm_weight is set      */
  int32_t row_gather;          /* 0: token tiles read a permuted copy of x made by the
                                  dispatch stage (default); 1: they gather their gate/up
                                  operand rows from x with TMA row gathers (no copy; slower
                                  on B200, where four-row gathers cannot feed the MMA).
                                  The weight-stream form always reads the copy;
                                  MOE_BF16_INT8W returns MOE_ERR_UNSUPPORTED with 1.      */
  int32_t separate_combine;    /* 0: the down projection's epilogue sums each token's two
                                  expert rows (default; bf16 and int8 weights without the
                                  post-norm); 1: a separate combine kernel does it (same
                                  result bit for bit)                                     */
} moe_options_t;

/* Optional outputs for inspection; each is a device pointer or NULL.
 * Permuted order = token slots sorted stably by (expert, token). */
typedef struct {
  int32_t* idx;        /* [T, 2] chosen experts, slot 0 = larger logit      */
  float* gates;        /* [T, 2] their softmax probabilities                */
  int32_t* counts;     /* [E]    token slots per expert                     */
  int32_t* offsets;    /* [E+1]  exclusive prefix of counts                 */
  int32_t* perm_token; /* [2T]   token of each permuted row                 */
  int32_t* perm_slot;  /* [2T]   slot (0/1) of each permuted row            */
  void* h;             /* [2T, f] GELU(x.Wg)*(x.Wu) per permuted row: x-dtype,
                          but fp16 for MOE_BF16_INT8W; when set, the kernels
                          write the intermediate here                         */
} moe_debug_t;

/* Passage: grok-field-guide "Grok-1 blueprint", section "MoE sublayer" (router,
 * top-2, gated experts, gate-weighted sum); gates as in Grok-1 book ch. 10,
 * section 10.3.1 (not renormalised); experts as in section 10.4 (GeGLU).
 * Forward pass with a library-owned workspace: one cache per device, grown
 * with cudaMalloc when a call needs more (never shrunk), guarded by a mutex.
 * Calls on one device share that workspace, so calls that may overlap on the
 * GPU (different streams) must use moe_forward_ex with their own workspaces.
 * Returns MOE_OK or an error status (see the file header). */
MOE_EXPORT moe_status_t moe_forward(const void* x, const float* w_router, const void* w_gate,
                         const void* w_up, const void* w_down,
                         const moe_scales_t* w_scales, void* out,
                         int64_t T, int64_t d, int64_t f, int32_t E, int32_t k,
                         moe_dtype_t dtype, moe_stream_t stream);

/* Passage: Grok-1 book ch. 11, section 11.3.1 item 3 (the sparse reorder and
 * grouped GEMM that replace the dense one-hot evaluation need the permuted
 * rows and intermediates this workspace holds).
 * Bytes of device workspace moe_forward_ex needs for these sizes with the
 * automatic kernel choices (path MOE_PATH_AUTO, automatic split-K), 0 on bad
 * arguments or T == 0. 256-byte multiple. Host only: no CUDA call. */
MOE_EXPORT size_t moe_workspace_size(int64_t T, int64_t d, int64_t f, int32_t E, int32_t k,
                                     moe_dtype_t dtype);

/* The same for a call whose moe_options_t sets `path` and `down_splits`
 * (0 = automatic), which change the workspace layout: 0 also when the split
 * factor does not divide f / 64 or the path is unknown. */
MOE_EXPORT size_t moe_workspace_size_ex(int64_t T, int64_t d, int64_t f, int32_t E, int32_t k,
                                        moe_dtype_t dtype, moe_path_t path, int32_t down_splits);

/* ---- Expert parallelism ----------------------------------------------------
 * Passage: Grok-1 book ch. 1, section 1.6.3 (the MoE layer shards the expert
 * axis over the devices of a (1, 8) mesh with shard_map). Building blocks of
 * that form on W GPUs, one process each, GPU r owning n = 8 / W consecutive
 * experts: each GPU routes and dispatches its own tokens (moe_route_dispatch;
 * the permuted rows are then grouped by owning GPU, because the permutation is
 * expert-major), the caller's communication library sends every block of rows
 * to its owner, the owner makes the received rows expert-contiguous
 * (moe_gather_rows), runs its experts on them (moe_experts_forward, which
 * also applies each row's gate), the rows go back the same way, and each GPU
 * sums its tokens' two rows (moe_combine). With the same split-K factor the
 * result equals moe_forward_ex's bit for bit. Every pointer is a device
 * pointer; workspaces are 256-byte aligned device memory of at least the
 * stated size; each call records its status word at the start of its
 * workspace (moe_device_status reads it). */

/* Outputs of moe_route_dispatch (device arrays owned by the caller). */
typedef struct {
  int32_t* idx;        /* [T, 2] chosen experts, slot 0 = larger logit          */
  float* gates;        /* [T, 2] their gates                                     */
  int32_t* counts;     /* [8]    token slots per expert                          */
  int32_t* offsets;    /* [9]    exclusive prefix of counts                      */
  int32_t* perm_token; /* [2T]   token of each permuted row                      */
  int32_t* perm_slot;  /* [2T]   slot of each permuted row                       */
  int32_t* slot_pos;   /* [T, 2] permuted row of each (token, slot)              */
  float* gate_perm;    /* [2T]   gate of each permuted row                       */
  void* xp;            /* [2T, d] x rows in permuted order: x's dtype, but fp16
                          for MOE_BF16_INT8W (the int8-weight GEMMs' operand)    */
} moe_routed_t;

/* Workspace bytes of moe_route_dispatch (0 on bad sizes or T == 0). */
MOE_EXPORT size_t moe_route_workspace_size(int64_t T, int64_t d, moe_dtype_t dtype);

/* The router and dispatch stages of moe_forward on T tokens: logits, softmax,
 * top-2 (gates renormalised if renormalize == 1), counts, offsets, the stable
 * (expert, token) permutation and the permuted copy of x. Same size limits
 * and errors as moe_forward_ex. */
MOE_EXPORT moe_status_t moe_route_dispatch(const void* x, const float* w_router, const float* router_bias,
                                           int64_t T, int64_t d, moe_dtype_t dtype, int32_t renormalize,
                                           const moe_routed_t* routed, void* workspace, size_t ws_bytes,
                                           moe_stream_t stream);

/* Rows for n_experts experts held by this GPU (row block e belongs to local
 * expert e, in order). */
typedef struct {
  const void* xp;              /* [R, d] rows, expert-contiguous: bf16 (MOE_BF16), fp16
                                  (MOE_BF16_INT8W) or fp32 (MOE_F32)                  */
  const int32_t* counts;       /* [n_experts] rows of each local expert (device)      */
  const float* gate;           /* [R] gate of each row, or NULL for 1                 */
  const void* w_gate;          /* [n_experts, d, f]                                   */
  const void* w_up;            /* [n_experts, d, f]                                   */
  const void* w_down;          /* [n_experts, f, d]                                   */
  const moe_scales_t* w_scales;/* MOE_BF16_INT8W: [n_experts, f], [n_experts, f],
                                  [n_experts, d]; else NULL                           */
  float* y;                    /* [R, d] fp32: gate * FFN_e(row)                       */
  int64_t R, d, f;
  int32_t n_experts;           /* 1 .. 8 */
  moe_dtype_t dtype;
} moe_expert_rows_t;

/* Workspace bytes of moe_experts_forward (0 on bad sizes, R == 0 or a split
 * factor that does not divide f / 64). `path` and `down_splits` as in
 * moe_options_t. */
MOE_EXPORT size_t moe_experts_workspace_size(int64_t R, int64_t d, int64_t f, int32_t n_experts,
                                             moe_dtype_t dtype, moe_path_t path, int32_t down_splits);

/* The expert GEMMs of moe_forward on rows already grouped by expert:
 * y[r] = gate[r] * down(act(xp[r] . w_gate[e]) * (xp[r] . w_up[e])) for the
 * rows r of local expert e (section 10.4 of ch. 10; activation, path and
 * down_splits from opts, NULL = defaults). Token-tile rows run on single CTAs
 * unless opts->path is MOE_PATH_TOKEN_TILE (CTA pairs). */
MOE_EXPORT moe_status_t moe_experts_forward(const moe_expert_rows_t* rows, const moe_options_t* opts,
                                            void* workspace, size_t ws_bytes, moe_stream_t stream);

/* out[t] = y[slot_pos[t,0]] + y[slot_pos[t,1]] (fp32 sum, in that order, then
 * cast to the x dtype: fp32 for MOE_F32, else bf16), with the post-RMSNorm
 * and residual add of moe_options_t when post_norm_weight / residual are set
 * (the blueprint's gate-weighted sum; ch. 10, section 10.3.1 sandwich norm).
 * y is [2T, d] fp32 in permuted order. Workspace: at least 256 bytes. */
MOE_EXPORT moe_status_t moe_combine(const float* y, const int32_t* slot_pos, int64_t T, int64_t d,
                                    moe_dtype_t dtype, const void* residual, const float* post_norm_weight,
                                    float norm_eps, void* out, void* workspace, size_t ws_bytes,
                                    moe_stream_t stream);

/* No counterpart on the pages (data movement of the expert-parallel form):
 * dst row i = src row index[i] (int32, device), for i < n; rows of row_bytes
 * bytes, a multiple of 4 (src and dst 4-byte aligned) or of 16 (16-byte
 * aligned, copied in 16-byte vectors); src has src_rows rows. Workspace: at
 * least 256 bytes. */
MOE_EXPORT moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int32_t* index, int64_t n,
                                        int64_t row_bytes, void* dst, void* workspace, size_t ws_bytes,
                                        moe_stream_t stream);

/* Passage: as moe_forward; the options follow Grok-1 book ch. 10, section
 * 10.3.1 (Mixtral renormalisation, sandwich post-norm) and section 10.4 (SiLU).
 * Forward pass on a caller-provided device workspace of ws_bytes bytes
 * (256-byte aligned, at least moe_workspace_size(...)); allocates nothing.
 * `opts` and `dbg` may be NULL. Concurrent calls need distinct workspaces. */
MOE_EXPORT moe_status_t moe_forward_ex(const moe_args_t* args, const moe_options_t* opts,
                            const moe_debug_t* dbg, void* workspace, size_t ws_bytes,
                            moe_stream_t stream);

/* Forward pass that allocates nothing: its scratch is a fixed 32 MiB device
 * array owned by the library (one per device that loads it, held until the
 * process exits). For callers that must not call cudaMalloc at run time, such
 * as a framework that reserves all device memory in its own pool at start-up,
 * or a latency-critical loop where an allocation would stall the device. The
 * pages have no counterpart: this is a deployment variant of moe_forward_ex.
 * Same arguments and results as moe_forward_ex without workspace and debug
 * outputs. With opts->down_splits == 0 the split-K factor is lowered until the
 * scratch fits. Returns MOE_ERR_WORKSPACE when the problem needs more than the
 * 32 MiB maximum (e.g. T = 64 at d = 6144, f = 32768 fits; T = 4096 does not).
 * The first call on a device looks up the array's device address and should
 * come before any stream capture; a call with T == 0 does only that set-up and
 * launches nothing. All calls on a device share the array: calls that may
 * overlap on the GPU race and must be ordered by the caller. The kernels'
 * status word lives in the array; moe_device_status(NULL, ...) reads it. */
MOE_EXPORT moe_status_t moe_forward_noalloc(const moe_args_t* args, const moe_options_t* opts,
                                            moe_stream_t stream);

/* No counterpart on the pages: the library's own failure reporting.
 * Synchronises `stream` and reads the status word that the kernels of the last
 * call on `workspace` recorded. With workspace == NULL it reads the two
 * library-owned words of the current device, the moe_forward cache's and the
 * moe_forward_noalloc scratch's (each if it exists), and reports their OR.
 * Returns MOE_OK, MOE_ERR_DEVICE_CHECK (and the raw code in *code if
 * code != NULL) or MOE_ERR_CUDA. */
MOE_EXPORT moe_status_t moe_device_status(const void* workspace, moe_stream_t stream, uint32_t* code);

/* Check of the failure path, with no fault: launches one thread that waits,
 * with the same bounded mbarrier wait the GEMM pipelines use, on a barrier that
 * nothing arrives on, giving up after `limit_us` microseconds (1 .. 10^7). The
 * kernel then records bit 0x10 in the status word at the start of `workspace`
 * (device memory, 256-byte aligned, at least 256 bytes) and returns, so a
 * following moe_device_status(workspace, stream, &code) returns
 * MOE_ERR_DEVICE_CHECK with code 0x10 and the context stays usable. No
 * counterpart on the pages: it exercises the library's own time limits.
 * Returns MOE_OK once launched, MOE_ERR_WORKSPACE / MOE_ERR_INVALID_ARG on bad
 * arguments, MOE_ERR_CUDA if the launch fails. */
MOE_EXPORT moe_status_t moe_selftest_bounded_wait(void* workspace, uint32_t limit_us, moe_stream_t stream);

/* No counterpart on the pages. Static description of a status code (never NULL). */
MOE_EXPORT const char* moe_status_string(moe_status_t status);

/* No counterpart on the pages. Library ABI version, currently 2. */
MOE_EXPORT int32_t moe_abi_version(void);

/* No counterpart on the pages. Options the library was compiled with, as bits:
 * MOE_BUILD_DEBUG_BOUNDS = the MOE_DEBUG_BOUNDS build (every index that one
 * kernel computes and another uses is checked before the access; a failed
 * check sets status bit 0x40 and skips the access; slower, for testing). */
#define MOE_BUILD_DEBUG_BOUNDS 1
MOE_EXPORT int32_t moe_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
