/*
 * mok.h -- C ABI of the forward Mixture-of-Kittens (MoK) MoE layer on one
 * B200 (sm_100a).
 *
 * The layer (MoK article on tahou.com, routing paragraph and the benchmark
 * paragraph listing "scheduling, dispatch, expert FFN, combine, weighted
 * merge"; MoK wiki summary "Mixture-of-Kittens: Cursor가 새로 공개한 NVL72용
 * MoE 학습 메가커널", key points) runs in five steps:
 *   1. router top-k over fp32 logits with softmax gates and a per-expert
 *      histogram;
 *   2. a device-built pull schedule {src_rank, src_index} per row of the
 *      expert-major layout (no sort, no host round trip);
 *   3. pull dispatch: a gather of token rows from R source shards into an
 *      expert-contiguous buffer;
 *   4. a grouped GEMM per expert with SwiGLU fused: h = silu(x Wg) * (x Wu),
 *      o = h Wd; the result row is pushed back to its token slot;
 *   5. the fixed-order weighted combine y[t] = sum_j g[t,j] o[t,j].
 *
 * Conventions for every call below:
 *  - Every data pointer is a DEVICE pointer owned by the caller unless the
 *    argument says "host".  The library never allocates device memory on
 *    these paths: scratch space is a caller-provided workspace whose size
 *    the matching *_workspace_bytes() call returns.  Workspaces must be
 *    256-byte aligned.
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream).  No call synchronises the host except
 *    mok_get_status(), mok_minibatch_bounds() and the *_host() calls.
 *  - Inputs are never modified.
 *  - Return value: MOK_OK or a MOK_ERR_* code; mok_last_error_string()
 *    gives a message for the calling thread's last failure.  Argument and
 *    shape errors are detected on the host before anything is enqueued.
 *  - Device-side failures (a bounded wait that gave up, a capacity bound)
 *    are written to a status word in the forward workspace and read with
 *    mok_get_status().
 *  - Layouts are row-major.  bf16 is IEEE bfloat16 stored as uint16.
 *  - Shapes: T tokens, H hidden, I expert intermediate, E experts, k top-k,
 *    R logical source shards; shard r holds tokens [r*S_r, (r+1)*S_r),
 *    S_r = T / R.  A "slot" is (t, j), j the rank in t's top-k list, slot
 *    index t*k + j; N_s = T*k slots.  A "row" is a position in the
 *    expert-major layout: rows offsets[e] .. offsets[e+1]-1 belong to
 *    expert e, in ascending token order.
 */
#ifndef MOK_H
#define MOK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mok_stream_t; /* same type as cudaStream_t */

enum {
    MOK_OK = 0,
    MOK_ERR_INVALID_ARG = 1, /* null pointer, negative size, k > E, ...      */
    MOK_ERR_UNSUPPORTED = 2, /* shape or alignment outside what is built     */
    MOK_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small   */
    MOK_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed            */
    MOK_ERR_TIMEOUT = 5,     /* a device-side wait gave up (device status)   */
    MOK_ERR_CAPACITY = 6     /* a device-side capacity bound was exceeded    */
};

enum { MOK_MAX_SHARDS = 64, MOK_MAX_EXPERTS = 1024, MOK_MAX_TOPK = 32 };

/* Form of the per-slot expert outputs out [T, k, H] that the grouped GEMM
 * pushes and the combine reads:
 *   MOK_SLOTS_F16S  the bf16 path: [N_s, H] fp16 values v and, at byte
 *                   offset mok_slot_exp_offset(N_s, H) of the same buffer,
 *                   [N_s, H/128] int8 exponents s, one per 128-feature block
 *                   of a row; the element is v * 2^s.  s puts the block's
 *                   largest magnitude in [2^14, 2^15) (clamped to
 *                   [-126, 126]), so a slot row keeps fp16's 11 significant
 *                   bits with fp32's exponent range;
 *   MOK_SLOTS_BF16  the MXFP8 path: [N_s, H] bf16;
 *   MOK_SLOTS_F32   [N_s, H] fp32 (accepted by mok_combine). */
enum { MOK_SLOTS_F32 = 0, MOK_SLOTS_BF16 = 1, MOK_SLOTS_F16S = 2 };

/* Bytes of a slot buffer of n_slots rows in the given form, and the byte
 * offset of the exponents of the MOK_SLOTS_F16S form (a multiple of 256). */
size_t mok_slot_bytes(int n_slots, int H, int slot_type);
size_t mok_slot_exp_offset(int n_slots, int H);

/* ------------------------------------------------------------------------
 * Step 1 + 2: the plan.
 * ---------------------------------------------------------------------- */

/* Views into the plan workspace, filled by mok_plan().  All device arrays.
 * A caller of mok_plan_noalloc fills one by hand from the arrays it passed
 * there (and T, E, k, R); the forward accepts it like mok_plan's. */
typedef struct mok_plan_t {
    int32_t T, E, k, R;
    int32_t* counts;          /* [E]   tokens routed to expert e              */
    int32_t* offsets;         /* [E+1] exclusive prefix sum; offsets[E]=N_s   */
    int32_t* sched_src_rank;  /* [N_s] per row: source shard  = t / S_r       */
    int32_t* sched_src_index; /* [N_s] per row: index in shard = t % S_r      */
    int32_t* row_slot;        /* [N_s] per row: slot t*k + j it came from      */
    int32_t* pos;             /* [N_s] per slot: its row                       */
    int32_t* topk_idx;        /* [T,k] selected experts in rank order          */
    float* gates;             /* [T,k] softmax over the k selected logits      */
} mok_plan_t;

/* Bytes of plan workspace for (T, E, k); 0 if the shape is invalid. */
size_t mok_plan_workspace_bytes(int T, int E, int k);

/*
 * mok_plan -- router top-k, gates, histogram and pull schedule.
 * Source: MoK article, routing paragraph (count each expert's tokens, plan
 * where they go, lay an expert's tokens out contiguously) and pull
 * paragraph (the destination needs only the source rank and the offset);
 * MoK wiki summary, schedule bullet ({src_rank, src_index} built on the
 * device, no sort, no CPU-GPU traffic).
 *   logits  [T, E] fp32, finite (NaN compares as -inf; order then unspecified)
 *   top_k   1 <= top_k <= min(E, MOK_MAX_TOPK);  E <= MOK_MAX_EXPERTS
 *   R       1 <= R <= MOK_MAX_SHARDS, T % R == 0
 *   ws      plan workspace (>= mok_plan_workspace_bytes), owned by the caller
 *   plan    host struct receiving views into ws; valid while ws lives
 * Selection: the k largest logits, ties to the lower expert index, listed in
 * rank order.  Gates: g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0).
 * Counts, offsets, schedule, row_slot and pos are deterministic (a stable
 * counting placement: ascending token inside each expert segment).
 */
int mok_plan(const float* logits, int T, int E, int top_k, int R,
             void* ws, size_t ws_bytes, mok_plan_t* plan, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * Step 1 with the router projection on the device.
 * ---------------------------------------------------------------------- */

enum { MOK_ROUTER_MAX_EXPERTS = 384 };

/* Bytes of EACH of the two router weight parts made by mok_router_prepare:
 * [E rounded up to 64, H] bf16.  0 for an unsupported shape. */
size_t mok_router_weights_bytes(int H, int E);

/*
 * mok_router_prepare -- one-time split of the router weights W_r [H, E]
 * fp32 (device) into two bf16 parts [E_pad, H] (expert-major, H
 * contiguous; E_pad = E rounded up to 64, padding rows zero):
 * w_hi = bf16(W_r), w_lo = bf16(W_r - w_hi), so w_hi + w_lo carries about
 * 16 significant bits of W_r with fp32's exponent range.  H % 64 == 0,
 * E <= MOK_ROUTER_MAX_EXPERTS; w_hi and w_lo (device, caller-owned,
 * mok_router_weights_bytes each) 16-byte aligned.  Asynchronous.
 */
int mok_router_prepare(const float* w_r, int H, int E, void* w_hi, void* w_lo, mok_stream_t stream);

/*
 * mok_plan_router -- mok_plan with the router projection computed on the
 * device: logits[t, e] = sum_h x[t, h] W_r[h, e] + prior[e], on the tensor
 * cores as x w_hi + x w_lo with fp32 accumulation, then the same top-k,
 * gates, histogram and pull schedule as mok_plan, in one router kernel
 * (projection, top-k and gates fused) plus the schedule kernels.
 * Source: MoK article, routing paragraph (a router assigns every token to
 * its experts; the projection is the plain reading the oracle's router
 * follows); MoK wiki summary, schedule bullet (the schedule is built on the
 * device without CPU traffic).
 *   x_shards    HOST array of R device pointers, shard r = [S_r, H] bf16
 *   w_hi, w_lo  from mok_router_prepare
 *   prior       [E] fp32 added to every token's logits, or NULL
 *   logits_out  [T, E] fp32 device array that receives the logits, or NULL
 *   ws, plan    as for mok_plan (same workspace size)
 * The logits differ from the exact projection by about 2^-17 + (H/16) 2^-23
 * of sum_h |x[t,h] W_r[h,e]| at most (the split, then one fp32 accumulator
 * addition per 16-wide MMA); logits closer than that may
 * be ordered either way (ties in the computed values still go to the lower
 * index).  A device-side failure (a bounded wait that gave up) is recorded
 * in the plan workspace's status word: mok_get_status(ws, ...) reads it
 * (mok_plan does not write that word).  Asynchronous on `stream`.
 */
int mok_plan_router(const void* const* x_shards, int H, const void* w_hi, const void* w_lo,
                    const float* prior, int T, int E, int top_k, int R, float* logits_out,
                    void* ws, size_t ws_bytes, mok_plan_t* plan, mok_stream_t stream);

/* Size of the library-owned scratch array used by mok_plan_noalloc. */
#define MOK_PLAN_NOALLOC_SCRATCH_BYTES (2u << 20)

/*
 * mok_plan_noalloc -- mok_plan for callers that cannot allocate device
 * memory: code recording a stream capture (allocation is not allowed
 * there), allocator-less runtimes that only hand out pre-registered
 * buffers, or hooks that must not touch the device allocator.  The paper
 * has no counterpart; this is a convenience of this library.
 *   Same inputs and the same results as mok_plan, bit for bit, but the
 *   caller passes the eight output arrays directly (device memory it owns:
 *   counts [E], offsets [E+1], sched_src_rank / sched_src_index / row_slot /
 *   pos / topk_idx [T*k] int32, gates [T*k] fp32) and no workspace.
 *   The plan's internal scratch lives in one static device array of
 *   MOK_PLAN_NOALLOC_SCRATCH_BYTES (2 MiB) inside the library, held by
 *   every GPU that loads the library until the process exits.  A shape is
 *   accepted when 4*T*k + 4*ceil(T/256)*E bytes (each part rounded up to
 *   256) fit in it, e.g. T*k up to about 440k slots at E = 384, k = 8
 *   (T = 16384, k = 8, E = 256 uses 576 KiB); larger
 *   shapes return MOK_ERR_UNSUPPORTED with a message (use mok_plan).
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library
 *   routine is called.  The first call on a device looks up the array's
 *   device address (cudaGetSymbolAddress, with that device current); make
 *   that first call before any stream capture.  The looked-up address is
 *   kept for the life of the process and belongs to the device's primary
 *   context (the one the CUDA runtime uses): after cudaDeviceReset, or when
 *   the calling thread has another context of that device current, it is
 *   stale, so do not call this entry point then.
 *   All calls on one device share the array: calls whose kernels may run at
 *   the same time on the GPU (unordered streams) race on it.  Every call
 *   writes each scratch entry before reading it, so no clearing is needed.
 *   Asynchronous on `stream`; errors as for mok_plan.
 */
int mok_plan_noalloc(const float* logits, int T, int E, int top_k, int R,
                     int32_t* counts, int32_t* offsets, int32_t* sched_src_rank,
                     int32_t* sched_src_index, int32_t* row_slot, int32_t* pos,
                     int32_t* topk_idx, float* gates, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * Steps 3-5: the forward layer.
 * ---------------------------------------------------------------------- */

enum {
    MOK_MODE_PERSISTENT = 0, /* one SM-partitioned persistent launch, ring    */
    MOK_MODE_STAGED = 1      /* gather, gate/up GEMM, down GEMM, combine as   */
                             /* four launches over full-size buffers          */
};

typedef struct mok_fwd_opts {
    int32_t mode;          /* MOK_MODE_*                                        */
    int32_t ring_slots;    /* rows of the ring token buffer (persistent mode);  */
                           /* 0 = 2 * max(minibatch, 4096) rows                 */
    int32_t dispatch_ctas; /* CTAs doing the dispatch in persistent mode;       */
                           /* 0 = default (6 bf16: bulk copies; 16 MXFP8:      */
                           /* quantising warps).  Every CTA combines once its  */
                           /* own role is done.  Must be 0 with dispatch_warps */
    int32_t gemm_ctas;     /* GEMM CTAs; 0 = all remaining SMs                  */
    int32_t mxfp8;         /* 1 = MXFP8 path (weights from                      */
                           /* mok_quantize_weights_mxfp8; either mode);         */
                           /* 0 = bf16                                          */
    int32_t min_waves;     /* persistent mode: a minibatch holds at least this  */
                           /* many full waves of gate/up units of the GEMM     */
                           /* CTAs; 0 = 2 (the pages' rule); < 0 = no floor    */
    int32_t save_for_backward; /* staged bf16 path: 1 = keep the gate and up    */
                           /* pre-activations (bf16) in the workspace for      */
                           /* mok_moe_backward                                 */
    int32_t dispatch_warps; /* persistent mode, 1 or 2: no dispatch CTAs; every */
                           /* CTA runs the GEMM and this many dispatch warps,  */
                           /* which claim the expert-major rows 16 at a time   */
                           /* and copy (MXFP8: quantise) them into the ring;   */
                           /* they combine once the rows are all claimed.      */
                           /* 0 = dispatch CTAs (dispatch_ctas)                */
    uint64_t timeout_ns;   /* bound on every device-side wait; 0 = 2 s          */
} mok_fwd_opts;

/* MXFP8 weight pack (opts->mxfp8 = 1): pass a pointer to this HOST struct
 * as mok_moe_forward's w_gate (w_up and w_down are then ignored).  Every
 * member is a device pointer made by mok_quantize_weights_mxfp8. */
typedef struct mok_mxfp8_weights {
    const void* gate;         /* [E, H, I] E4M3      */
    const void* gate_scales;  /* [E, H/32, I] E8M0   */
    const void* up;           /* [E, H, I] E4M3      */
    const void* up_scales;    /* [E, H/32, I] E8M0   */
    const void* down;         /* [E, I, H] E4M3      */
    const void* down_scales;  /* [E, I/32, H] E8M0   */
} mok_mxfp8_weights;

/* Bytes of forward workspace; 0 if the shape is invalid.  opts may be NULL
 * (defaults).  minibatch = rows per minibatch (see mok_moe_forward). */
size_t mok_forward_workspace_bytes(int T, int H, int I, int E, int k, int minibatch,
                                   const mok_fwd_opts* opts);

/*
 * mok_moe_forward -- pull dispatch, expert FFN (SwiGLU), push combine and
 * the weighted merge.
 * Source: MoK article, pull paragraph (forward dispatch pulls), push-combine
 * paragraph (results are pushed back to their token's slot), megakernel and
 * minibatch paragraphs (SM split, local counters, at least two waves per
 * minibatch), ring-buffer paragraph (fixed-size token buffer reused once the
 * combine has shipped a minibatch's results), benchmark paragraph (weighted
 * merge); MoK wiki summary, key points (SM split, TMA, local counters).
 *   x_shards  HOST array of R device pointers, shard r = [S_r, H] bf16
 *   H, I      hidden and intermediate sizes; H % 128 == 0, I % 64 == 0
 *   w_gate    [E, H, I] bf16
 *   w_up      [E, H, I] bf16
 *   w_down    [E, I, H] bf16
 *   plan      from mok_plan() on the same stream (its workspace must live)
 *   minibatch persistent mode: the least rows of the expert-major layout
 *             per minibatch (>= 16), or 0 for the two-wave rule alone.  A
 *             minibatch ends at the first expert boundary where it holds
 *             at least `minibatch` rows and opts->min_waves (default 2)
 *             full waves of gate/up units for the GEMM CTAs, or at half
 *             the ring (an expert taller than that is split).  Ignored in
 *             staged mode (one minibatch).
 *   opts      may be NULL (persistent mode, defaults)
 *   ws        forward workspace (>= mok_forward_workspace_bytes)
 *   y_shards  HOST array of R device pointers, shard r = [S_r, H] bf16
 * Arithmetic: gate/up in bf16 x bf16 with fp32 accumulation; h =
 * silu(gate) * up rounded once to bf16; down projection bf16 x bf16 with
 * fp32 accumulation; each expert output row stored fp32 at its slot;
 * y[t] = bf16(sum_{j<k} g[t,j] * o[t,j]) accumulated in fp32 with j
 * ascending (one bf16 rounding of y).  No step saturates: every stored
 * intermediate has the exponent range of fp32.  y does not depend on the
 * mode, minibatch, ring size or R.
 * MXFP8 path (opts->mxfp8 = 1, either mode, w_gate = a mok_mxfp8_weights
 * HOST struct): x is quantised in the gather (persistent mode: by the
 * dispatch CTAs, into the ring) and h in the SwiGLU epilogue
 * (32-element blocks, E8M0 scale + E4M3 values, as mok_mxfp8_quantize_rows
 * does); both GEMMs run on the block-scaled E4M3 x E4M3 tensor-core MMA
 * with fp32 accumulation; slot outputs bf16 and the combine as above.
 */
int mok_moe_forward(const void* const* x_shards, int H, int I,
                    const void* w_gate, const void* w_up, const void* w_down,
                    const mok_plan_t* plan, int minibatch, const mok_fwd_opts* opts,
                    void* ws, size_t ws_bytes, void* const* y_shards, mok_stream_t stream);

/*
 * mok_two_wave_rows -- the two-wave minibatch size: the rows of the
 * expert-major layout whose gate/up output tiles (tile_rows rows x
 * tile_features of the 2I gate and up columns each) make two full waves of
 * `gemm_ctas` CTAs, ceil(2 * gemm_ctas * tile_rows * tile_features / (2 I)).
 * Source: MoK article, minibatch paragraph (a minibatch must fill at least
 * two waves of the GEMM SMs, about 2368 tokens at hidden 7168 /
 * intermediate 2048; that is 128 x 256 tiles over 148 SMs); MoK wiki
 * summary, minibatch bullet.  The forward's own units are chunks of up to
 * 256 rows x 128 features (256 with M-tile pairs), and it counts them on
 * the device (see mok_moe_forward's minibatch); this host formula gives the
 * rows that suffice when every chunk is full height.  Returns 0 for
 * non-positive arguments.
 */
int mok_two_wave_rows(int I, int gemm_ctas, int tile_rows, int tile_features);

/*
 * mok_minibatch_bounds -- the minibatches mok_moe_forward would use for
 * these arguments (persistent mode): builds the work list in `ws` exactly
 * as the forward does, synchronises `stream`, and writes to HOST arrays the
 * first row of each minibatch (row0) and, if `units` is not NULL, its
 * gate/up unit count; at most max_mb entries; *n_mb receives the number of
 * minibatches.  Arguments and errors as for mok_moe_forward (x and y are
 * not needed).  An inspection call: it synchronises the host.
 */
int mok_minibatch_bounds(const mok_plan_t* plan, int H, int I, const void* w_gate, int minibatch,
                         const mok_fwd_opts* opts, void* ws, size_t ws_bytes, int32_t* row0,
                         int32_t* units, int max_mb, int* n_mb, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * The backward of the layer (bf16 path).
 * ---------------------------------------------------------------------- */

/* Bytes of backward workspace: do rows [N_s, H] bf16, [da | db] rows
 * [N_s, 2I] bf16, dx rows [N_s, H] as MOK_SLOTS_F16S (fp16 values, one
 * exponent per 128 features) and a status word. */
size_t mok_backward_workspace_bytes(int T, int H, int I, int E, int k);

/*
 * mok_moe_backward -- gradients of the layer given dy.
 * Source: MoK article, the Pull/Push paragraph (the backward pairs a pull
 * reverse-combine with a push reverse-dispatch); the arithmetic is the
 * chain rule of the forward, step by step:
 *   1. pull reverse-combine: for each slot (t, j), do = g[t,j] dy_t as a
 *      bf16 row in the expert-major layout, dg[t,j] = <dy_t, o[t,j]>;
 *   2. dh = do Wd^T (fp32 accumulation); da = dh b silu'(a),
 *      db = dh silu(a), rounded to bf16;
 *   3. dx rows = da Wg^T + db Wu^T (fp32 accumulation), pushed to their
 *      token's slot as fp16 with one power-of-two exponent per 128 features;
 *   4. push reverse-dispatch: dx_t = bf16(sum_j dx rows of t), j ascending;
 *   5. dWd[e] = h^T do, dWg[e] = x^T da, dWu[e] = x^T db over the expert's
 *      rows (fp32 accumulation, bf16 results; an expert with no rows gets
 *      zeros);
 *   6. dlogits[t, sel[t,j]] = g[t,j] (dg[t,j] - sum_i g[t,i] dg[t,i]), 0 for
 *      unselected experts (the selection has no gradient).
 *   dy_shards  HOST array of R device pointers, shard r = [S_r, H] bf16
 *   w_*        the forward's bf16 weights
 *   plan       the forward's plan
 *   fwd_ws     the workspace of the staged mok_moe_forward call on this plan
 *              with opts.save_for_backward = 1 (it holds the gathered rows,
 *              h, the gate and up pre-activations a and b, and the fp32
 *              slot outputs o); not modified
 *   dx_shards  HOST array of R device pointers, shard r = [S_r, H] bf16
 *   dw_gate, dw_up [E, H, I] bf16; dw_down [E, I, H] bf16; dlogits [T, E] fp32
 *   ws         backward workspace (>= mok_backward_workspace_bytes)
 * H % 128 == 0, I % 128 == 0.  Device-side failures go to ws's status word
 * (mok_get_status).  Asynchronous on `stream`.
 */
int mok_moe_backward(const void* const* dy_shards, int H, int I,
                     const void* w_gate, const void* w_up, const void* w_down,
                     const mok_plan_t* plan, const void* fwd_ws, size_t fwd_ws_bytes,
                     void* const* dx_shards, void* dw_gate, void* dw_up, void* dw_down,
                     float* dlogits, void* ws, size_t ws_bytes, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * MXFP8 (OCP MX v1.0: 32-element blocks, E8M0 scale byte = s + 127 with
 * s = floor(log2(max|v|)) - 8 clamped to [-127, 127], an all-zero block
 * gets 0x00; E4M3 elements = v / 2^s rounded to nearest even, saturating at
 * +-448).  Source: MoK article, paragraph after the ring buffer (MXFP8
 * activation quantisation fused into dispatch, grouped GEMM and SwiGLU).
 * ---------------------------------------------------------------------- */

/* Activation layout: blocks of 32 consecutive elements along each row.
 *   src     [rows, K] bf16 (src_f32 = 0) or fp32 (src_f32 = 1); K % 32 == 0
 *   q       [rows, K] E4M3 bytes;  scales [rows, K/32] E8M0 bytes
 * This is the quantiser the MXFP8 forward fuses into the gather (x) and the
 * SwiGLU epilogue (h). */
int mok_mxfp8_quantize_rows(const void* src, int src_f32, int rows, int K, void* q, void* scales,
                            mok_stream_t stream);

/* Weight layout: w [E, K, N] bf16 (K = contraction index, N = output
 * columns, i.e. Wg/Wu with K = H, N = I and Wd with K = I, N = H); blocks of
 * 32 along K of each column.  q [E, K, N] E4M3 bytes (same layout as w),
 * scales [E, K/32, N] E8M0 bytes.  K % 32 == 0.  One-time, at weight load. */
int mok_quantize_weights_mxfp8(const void* w_bf16, int E, int K, int N, void* q, void* scales,
                               mok_stream_t stream);

/*
 * mok_get_status -- synchronise `stream` and read the device status word of
 * a forward workspace (or of a plan workspace after mok_plan_router).  *device_code receives MOK_OK, MOK_ERR_TIMEOUT or
 * MOK_ERR_CAPACITY; the return value is MOK_OK unless the read itself
 * failed.  The status word is cleared at the start of every forward.
 */
int mok_get_status(const void* ws, size_t ws_bytes, mok_stream_t stream, int* device_code);

/* Message for the calling thread's last non-OK return (never NULL). */
const char* mok_last_error_string(void);

/* ------------------------------------------------------------------------
 * The steps one at a time (parity bisection and per-kernel profiling).
 * They compute exactly what mok_moe_forward's staged mode computes.
 * ---------------------------------------------------------------------- */

/* rows[row] = x_shard[src_rank[row]][src_index[row]], row < plan->T*plan->k.
 * rows: [N_s, H] bf16.  Source: MoK article, pull paragraph. */
int mok_gather(const void* const* x_shards, int H, const mok_plan_t* plan,
               void* rows, mok_stream_t stream);

/* The MXFP8 gather (what mok_moe_forward's MXFP8 path runs): every row is
 * quantised in 32-element blocks as mok_mxfp8_quantize_rows does, in the
 * operand form of the block-scaled MMA:
 *   rows_q [N_s, H] E4M3 bytes, rows_q[row] = the blocks of the row's token;
 *   scales [H/128][sc_rows][4] E8M0 bytes: plane g, row r, byte b = the
 *     scale of block 4g + b of row r; sc_rows = mok_mxfp8_scale_rows(N_s).
 * H % 128 == 0; rows_q and scales 16-byte aligned.  Source: MoK article,
 * paragraph on MXFP8 activation quantisation inside the dispatch. */
int mok_mxfp8_scale_rows(int n_rows);
int mok_gather_mxfp8(const void* const* x_shards, int H, const mok_plan_t* plan,
                     void* rows_q, void* scales, mok_stream_t stream);

/* Bytes of scratch for mok_expert_ffn. */
size_t mok_expert_ffn_workspace_bytes(int n_rows, int I, int E);

/* Grouped SwiGLU FFN over the expert-major rows of `plan`:
 *   h[row]   = bf16(silu(rows[row] Wg[e]) * (rows[row] Wu[e]))   [N_s, I]
 *   out[row_slot[row]] = h[row] Wd[e]  (fp32 accumulation)       [N_s, H]
 * (e = expert of the row; all weights bf16).  h stays in the workspace;
 * `out` is slot-indexed ([T, k, H]) in the MOK_SLOTS_F16S form: a buffer of
 * mok_slot_bytes(N_s, H, MOK_SLOTS_F16S) bytes, 256-byte aligned, whose
 * fp32 results are stored as fp16 values with one exponent per 128
 * features (the form mok_moe_forward's bf16 path pushes).  Source: MoK
 * article, routing paragraph (grouped GEMM over contiguous per-expert
 * tokens) and push-combine paragraph. */
int mok_expert_ffn(const void* rows, int H, int I,
                   const void* w_gate, const void* w_up, const void* w_down,
                   const mok_plan_t* plan, void* ws, size_t ws_bytes,
                   void* out, mok_stream_t stream);

/* Bytes of scratch for mok_expert_ffn_mxfp8. */
size_t mok_expert_ffn_mxfp8_workspace_bytes(int n_rows, int I, int E);

/* The grouped SwiGLU FFN of the MXFP8 path (block-scaled tensor-core MMA)
 * over the output of mok_gather_mxfp8 (rows_q, scales; same layouts), with
 * the weight pack `w` (host struct) of mok_quantize_weights_mxfp8.  h is
 * quantised to MXFP8 in the SwiGLU epilogue and stays in the workspace;
 * out: [T, k, H] bf16 (MOK_SLOTS_BF16), slot-indexed.  Source: MoK
 * article, paragraph on MXFP8 inside the GEMM and SwiGLU. */
int mok_expert_ffn_mxfp8(const void* rows_q, const void* scales, int H, int I,
                         const mok_mxfp8_weights* w, const mok_plan_t* plan,
                         void* ws, size_t ws_bytes, void* out, mok_stream_t stream);

/* y[t] = bf16(sum_{j<k} gates[t,j] * out[t,j,:]), fp32, j ascending,
 * written to y_shard[t / S_r][t % S_r].  out: [T, k, H] in the form
 * out_dtype names (MOK_SLOTS_F32, MOK_SLOTS_BF16, or MOK_SLOTS_F16S with
 * H % 128 == 0), 16-byte aligned.
 * Source: MoK article, benchmark paragraph (final weighted merge). */
int mok_combine(const void* out, int out_dtype, int H, const mok_plan_t* plan,
                void* const* y_shards, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * End to end from host memory (what a caller without device buffers uses).
 * ---------------------------------------------------------------------- */

/* Bytes of workspace for mok_moe_forward_host. */
size_t mok_forward_host_workspace_bytes(int T, int H, int I, int E, int k, int minibatch,
                                        const mok_fwd_opts* opts);

/*
 * mok_moe_forward_host -- copies HOST x [T, H] bf16 and HOST logits [T, E]
 * fp32 to the device, runs mok_plan and mok_moe_forward, copies y [T, H]
 * bf16 back to HOST memory and synchronises `stream`.  Weights are device
 * pointers as in mok_moe_forward.  Host buffers should be pinned for
 * full copy bandwidth (pageable memory works, slower).  ws: device
 * workspace of mok_forward_host_workspace_bytes().
 */
int mok_moe_forward_host(const void* x_host, const float* logits_host,
                         int T, int H, int I, int E, int top_k, int R,
                         const void* w_gate, const void* w_up, const void* w_down,
                         int minibatch, const mok_fwd_opts* opts,
                         void* ws, size_t ws_bytes, void* y_host, mok_stream_t stream);

/* Bytes of workspace for mok_moe_forward_host_batches: two sets of device
 * staging buffers (x, y, logits), one plan and one forward workspace. */
size_t mok_forward_host_batches_workspace_bytes(int T, int H, int I, int E, int k, int minibatch,
                                                const mok_fwd_opts* opts);

/*
 * mok_moe_forward_host_batches -- n batches of T tokens through the layer
 * from HOST buffers, with the copies overlapped with the compute: batch i
 * uses device staging set i % 2, and while batch i computes on `stream`,
 * batch i+1's x and logits are uploaded and batch i-1's y is downloaded on
 * two other streams (one per copy direction).  x_host[i] [T, H] bf16,
 * logits_host[i] [T, E] fp32 and y_host[i] [T, H] bf16 are HOST arrays of
 * n pointers; pinned memory gives the overlap (pageable copies serialise).
 * Batch i's y_host[i] may be the same buffer as another batch's.  The
 * results equal n calls of mok_moe_forward_host, bit for bit.  Returns
 * after every copy has finished (synchronises `stream`); on an error, no
 * copy is left in flight.  The two copy streams and their events are made
 * on a device's first call and kept until the process exits; calls on one
 * device run one at a time (a mutex).  (This serves the pages' data path
 * from host memory; the pages have no counterpart of the call itself.)
 */
int mok_moe_forward_host_batches(int n, const void* const* x_host, const float* const* logits_host,
                                 void* const* y_host, int T, int H, int I, int E, int top_k, int R,
                                 const void* w_gate, const void* w_up, const void* w_down,
                                 int minibatch, const mok_fwd_opts* opts,
                                 void* ws, size_t ws_bytes, mok_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism over G GPUs, one process per GPU.
 * Source: MoK article, pull-dispatch paragraph (the rank that owns an expert
 * pulls that expert's tokens from the source ranks' memory by
 * {src_rank, src_index}) and push-combine paragraph (each expert output goes
 * back to its token's rank, which merges its k results); MoK wiki summary,
 * key points (NVLink loads and stores from inside the kernels, no
 * collective library on the data path).
 *
 * Rank g holds tokens [g*S_r, (g+1)*S_r) of the layer (S_r = T / G) in its
 * x buffer and the experts [e0, e0 + e_loc) (the weights of those experts
 * only).  Every rank builds the same plan with mok_plan over the
 * all-gathered logits [T, E] with R = G, so the plan's source shard of a
 * token is its rank.  A step s = 1, 2, ... on every rank:
 *   mok_ep_dispatch_ffn(step s)  group barrier (every rank's x is ready and
 *                                every rank has finished reading its slot
 *                                buffer in step s-1), pull dispatch of this
 *                                rank's rows from the ranks' x over NVLink,
 *                                the grouped SwiGLU FFN, and the push of
 *                                every slot row into its token's rank's slot
 *                                buffer from the down GEMM's epilogue;
 *   mok_ep_combine(step s)       group barrier (every push of step s has
 *                                landed), then the fixed-order weighted
 *                                combine of this rank's tokens.
 * The results equal mok_moe_forward's staged path (bf16 or MXFP8) over the
 * same plan, bit for bit.
 * ---------------------------------------------------------------------- */

/* How the ranks of a group are ordered between the two calls of a step:
 *   MOK_EP_SYNC_DEVICE  each call starts with a device-side barrier over the
 *                       counters in the ranks' slot buffers (the multi-GPU
 *                       mode: one process per GPU, every wait bounded);
 *   MOK_EP_SYNC_CALLER  no barrier: the caller orders the ranks' calls (one
 *                       process driving every rank's buffers, e.g. all on
 *                       one GPU; all ranks' mok_ep_dispatch_ffn, then all
 *                       ranks' mok_ep_combine). */
enum { MOK_EP_SYNC_CALLER = 0, MOK_EP_SYNC_DEVICE = 1 };

typedef struct mok_ep_t {
    int32_t G;     /* ranks in the group, 1 .. MOK_MAX_SHARDS (the plan's R)  */
    int32_t g;     /* this rank, 0 .. G-1                                     */
    int32_t e0;    /* this rank's experts: e0 .. e0 + e_loc - 1 of the plan's */
    int32_t e_loc; /* E (e_loc may be 0)                                      */
    int32_t sync;  /* MOK_EP_SYNC_DEVICE or MOK_EP_SYNC_CALLER                */
    int32_t mxfp8; /* 0: bf16 path (mok_ep_dispatch_ffn, fp16 slot rows with  */
                   /* exponents); 1: MXFP8 path (mok_ep_dispatch_ffn_mxfp8,   */
                   /* bf16 slot rows)                                          */
    /* x[h]: rank h's tokens [S_r, H] bf16, as THIS GPU addresses them (a
     * peer pointer from mok_ipc_import, or a local pointer), 16-byte
     * aligned; h < G. */
    const void* x[MOK_MAX_SHARDS];
    /* slots[h]: rank h's slot buffer of mok_ep_slot_bytes(S_r, H, k) bytes,
     * as THIS GPU addresses it, 256-byte aligned; zero-filled once before
     * the group's first step (it holds the barrier counter). */
    void* slots[MOK_MAX_SHARDS];
} mok_ep_t;

/* Bytes of one rank's slot buffer: [S_r*k, H] fp16 slot rows with their
 * block exponents (the MOK_SLOTS_F16S form of mok_slot_bytes; the MXFP8
 * path stores bf16 rows [S_r*k, H] at its start), then the 256-byte barrier
 * counter region.  H % 128 == 0; 0 if the shape is invalid. */
size_t mok_ep_slot_bytes(int S_r, int H, int k);

/* Bytes of the per-rank workspace for (T, H, I, e_loc, k), either path:
 * status word, the local expert offsets, the work list, and room for every
 * slot's row and h row (a rank may receive all T*k rows). */
size_t mok_ep_workspace_bytes(int T, int H, int I, int e_loc, int k);

/*
 * mok_ep_dispatch_ffn -- the first half of an expert-parallel step on rank
 * ep->g: barrier (MOK_EP_SYNC_DEVICE), pull dispatch, grouped SwiGLU FFN and
 * push.
 *   plan      the group's plan (R == ep->G), identical on every rank
 *   w_gate    [e_loc, H, I] bf16, w_up [e_loc, H, I], w_down [e_loc, I, H]:
 *             the weights of experts e0 .. e0 + e_loc - 1 on this GPU
 *   step      1, 2, 3, ... (the same on every rank; the barrier waits for
 *             every rank's arrival number 2*step - 1)
 *   timeout_ns  bound of the barrier's wait (0: 2 s); a wait that gives up
 *             writes MOK_ERR_TIMEOUT to the workspace's status word
 *   ws        this rank's workspace (>= mok_ep_workspace_bytes(T, H, I,
 *             e_loc, k)); its status word is cleared at the start
 * H % 128 == 0, I % 64 == 0.  Asynchronous on `stream`.
 */
int mok_ep_dispatch_ffn(const mok_plan_t* plan, const mok_ep_t* ep, int H, int I,
                        const void* w_gate, const void* w_up, const void* w_down,
                        uint32_t step, uint64_t timeout_ns, void* ws, size_t ws_bytes,
                        mok_stream_t stream);

/*
 * mok_ep_dispatch_ffn_mxfp8 -- the same on the MXFP8 path (ep->mxfp8 == 1):
 * the pull quantises each row to E4M3 with its block scales (as
 * mok_gather_mxfp8), the grouped FFN runs on the block-scaled MMA (as
 * mok_expert_ffn_mxfp8) with `w`, the pack of mok_quantize_weights_mxfp8
 * for this rank's e_loc experts (host struct, device arrays), and the down
 * epilogue pushes bf16 slot rows.  The results equal mok_moe_forward's
 * staged MXFP8 path over the same plan, bit for bit.
 */
int mok_ep_dispatch_ffn_mxfp8(const mok_plan_t* plan, const mok_ep_t* ep, int H, int I,
                              const mok_mxfp8_weights* w, uint32_t step, uint64_t timeout_ns,
                              void* ws, size_t ws_bytes, mok_stream_t stream);

/*
 * mok_ep_combine -- the second half of step `step` on rank ep->g: barrier
 * (MOK_EP_SYNC_DEVICE; arrival number 2*step), then
 *   y[i] = bf16(sum_{j<k} gates[t,j] * out[t,j,:]),  t = g*S_r + i,
 * over the slot rows in this rank's slot buffer (ep->slots[ep->g]; fp16
 * with exponents, or bf16 when ep->mxfp8), fp32, j ascending.
 * y: [S_r, H] bf16, 16-byte aligned.  ws: the workspace given to the
 * dispatch call (its status word).  Asynchronous on `stream`.
 */
int mok_ep_combine(const mok_plan_t* plan, const mok_ep_t* ep, int H, uint32_t step,
                   uint64_t timeout_ns, void* y, void* ws, size_t ws_bytes, mok_stream_t stream);

/* CUDA IPC for the peer pointers of mok_ep_t.  mok_ipc_export writes the
 * MOK_IPC_HANDLE_BYTES-byte handle of the cudaMalloc allocation holding
 * `dptr` and dptr's byte offset in it; another process opens it with
 * mok_ipc_import (peer access enabled on demand; the allocation is then
 * addressed as *base + offset) and releases it with mok_ipc_close(base).
 * Memory from cudaMalloc (PyTorch's default allocator) only. */
#define MOK_IPC_HANDLE_BYTES 64
int mok_ipc_export(const void* dptr, void* handle, size_t* offset);
int mok_ipc_import(const void* handle, void** base);
int mok_ipc_close(void* base);

#ifdef __cplusplus
}
#endif
#endif /* MOK_H */
