/*
 * maple_moe.h -- C ABI of the B200 (sm_100a) ternary-weight mixture-of-experts
 * FFN layer.
 *
 * The layer is the expert FFN of the Maple-Preview 20B-A1B model: 256 experts
 * per layer, every token routed to its top 8 ("linlog.top/article/1232",
 * section 架构设计, model table), expert weights in {-alpha, 0, +alpha} with
 * one learned alpha per output row, so that each product becomes an add, a
 * subtract or a skip (same page, section 三值权重：把乘法变成加法).  The
 * pages give no interface; this one takes device pointers and a CUDA stream.
 *
 * Forward pass, per token t (x_t bf16 of length D):
 *   route:    logit_e = x_t . Wr_e (+ b_e), fp32, fixed summation order;
 *             keep the K largest (ties: lower expert index), w = softmax over
 *             the kept logits.
 *   quantise: q_x = int8 absmax codes of x_t, s_x = amax/127.
 *   per kept expert e:
 *             accG = Tgate_e q_x, accU = Tup_e q_x        (int32, exact)
 *             h    = SiLU(accG*alphaG*s_x) * (accU*alphaU*s_x)   (fp32)
 *             q_h, s_h = int8 absmax codes of h
 *             accD = Tdown_e q_h                           (int32, exact)
 *             yE   = accD * alphaD * s_h
 *   combine:  y_t = sum_k w_k yE_k  (rank order, fmaf from 0).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device unless
 *    stated otherwise, row-major, 16-byte aligned.  The caller owns them.
 *  - Every call is asynchronous on the given stream (NULL = legacy default
 *    stream) and never synchronises, except maple_moe_destroy.
 *  - Return value: MAPLE_OK (0) or a negative MAPLE_ERR_* code; nothing is
 *    printed, nothing aborts.  A kernel that meets an invalid value (a NaN
 *    router logit, an out-of-range expert id) sets a flag in host-mapped
 *    memory; the next call on the same handle returns MAPLE_ERR_DEVICE_FLAG
 *    (and clears it), and maple_moe_device_flags reads it on demand.
 *  - Every wait inside a kernel (on another warp, another CTA or a copy in
 *    flight) is bounded in time (2 s unless maple_moe_set_debug sets another
 *    limit).  A wait that gives up sets MAPLE_FLAG_TIMEOUT; the kernel drains
 *    its copies in flight and returns, and the outputs of that call are not
 *    valid.  The next call on the handle that sees the flag returns
 *    MAPLE_ERR_TIMEOUT, after resetting the handle's internal counters on its
 *    stream, so that the call after it runs normally.  Calls enqueued before
 *    the flag became visible to the host may be wrong as well; synchronise
 *    and check maple_moe_device_flags when that matters.
 *  - A handle may be used from one stream at a time.
 */
#ifndef MAPLE_MOE_H
#define MAPLE_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *maple_stream_t;   /* the same type as cudaStream_t */

typedef struct maple_moe_s *maple_moe_t;

enum {
    MAPLE_OK = 0,
    MAPLE_ERR_INVALID_ARG = -1,       /* NULL or misaligned pointer, T out of range, bad handle */
    MAPLE_ERR_UNSUPPORTED_SHAPE = -2, /* shape outside the limits listed at maple_moe_config */
    MAPLE_ERR_OOM = -3,               /* device allocation failed in create */
    MAPLE_ERR_CUDA = -4,              /* a CUDA runtime call or a kernel launch failed */
    MAPLE_ERR_TIMEOUT = -5,           /* an earlier call's bounded device wait gave up (MAPLE_FLAG_TIMEOUT) */
    MAPLE_ERR_DEVICE_FLAG = -6,       /* an earlier kernel on this handle flagged an invalid value */
};

/* device flag bits (maple_moe_device_flags) */
#define MAPLE_FLAG_NAN_LOGIT 0x1u     /* a router logit was NaN; it was ranked last */
#define MAPLE_FLAG_BAD_INDEX 0x2u     /* an expert id outside [0, E) reached the permutation */
#define MAPLE_FLAG_BAD_VALUE 0x4u     /* maple_moe_pack_ternary met a value outside {-1, 0, +1} */
#define MAPLE_FLAG_TIMEOUT 0x8u       /* a bounded wait inside a kernel gave up (reported as MAPLE_ERR_TIMEOUT) */

/* config.flags: path selection and weight layouts (default 0 = automatic, both layouts) */
#define MAPLE_CFG_FORCE_GEMV 0x1u     /* never use the tensor-core grouped GEMM: T <= 64 on the decode
                                         kernel whatever decode_max_tokens says, larger T rejected
                                         (MAPLE_ERR_UNSUPPORTED_SHAPE); only the decode layout is built */
#define MAPLE_CFG_FORCE_TC 0x2u       /* the tensor-core grouped GEMM for every T > 0; only its layout is
                                         built (may not be combined with the other flags) */
#define MAPLE_CFG_DECODE_ONLY 0x4u    /* build only the decode layout (half the weight memory);
                                         T > decode_max_tokens is rejected (MAPLE_ERR_UNSUPPORTED_SHAPE) */

/*
 * Layer shape.  Limits: d_model = 256 * 2^i (256 .. 4096); d_ff = 128 * 2^j
 * (128 .. 1024); n_experts % 16 == 0
 * and 16 <= n_experts <= 1024; 1 <= top_k <= min(32, n_experts);
 * 1 <= max_tokens <= 65536.  max_tokens sizes the library-owned workspace.
 * decode_max_tokens (0 .. 64, 0 selects 64): largest T served by the decode
 * kernel (weight streaming on warp-level int8 MMA); larger T use the tcgen05
 * int8 grouped GEMM.  The decode kernel needs d_ff <= d_model and its
 * shared memory to fit; shapes outside that run every T on the tensor cores
 * (and then reject MAPLE_CFG_FORCE_GEMV and MAPLE_CFG_DECODE_ONLY).
 */
typedef struct {
    int32_t d_model, n_experts, top_k, d_ff, max_tokens;
    int32_t decode_max_tokens;
    uint32_t flags;
} maple_moe_config;

/*
 * Weights in the 2-bit interchange format (maple_moe_pack_ternary writes it):
 * a row of n ternary values is n/16 uint32 words; value j sits in word j/16,
 * bits 2*(j%16) and 2*(j%16)+1; code 0 = 0, 1 = +1, 2 = -1 (3 reads as 0).
 * All DEVICE pointers, caller-owned; create copies what it needs, so they may
 * be freed once the stream passed to create has synchronised.
 */
typedef struct {
    const uint32_t *w_gate;      /* [E][F][D/16]  row r of expert e = output channel r */
    const uint32_t *w_up;        /* [E][F][D/16] */
    const uint32_t *w_down;      /* [E][D][F/16]  row c = output channel c */
    const float *alpha_gate;     /* [E][F]  one scale per output row */
    const float *alpha_up;       /* [E][F] */
    const float *alpha_down;     /* [E][D] */
    const float *router_w;       /* [E][D]  fp32 */
    const float *router_bias;    /* [E] or NULL */
} maple_moe_weights;

/*
 * Optional DEVICE outputs of the intermediate results of maple_moe_forward,
 * for checking.  Any field may be NULL.  "Slot" s = t*K + k is token t's k-th
 * choice; per-slot arrays are indexed by s.
 */
typedef struct {
    int8_t *q_x;            /* [T][D]   int8 codes of x */
    float *s_x;             /* [T]      scale of x */
    float *logits;          /* [T][E]   router logits */
    int32_t *topk_idx;      /* [T][K] */
    float *topk_w;          /* [T][K] */
    int32_t *acc_gate;      /* [T*K][F] int32 accumulators before scaling */
    int32_t *acc_up;        /* [T*K][F] */
    int8_t *q_h;            /* [T*K][F] int8 codes of the SwiGLU output */
    float *s_h;             /* [T*K] */
    int32_t *acc_down;      /* [T*K][D] */
    int32_t *expert_counts; /* [E] */
    int32_t *expert_offsets;/* [E+1]  exclusive prefix sum of the counts */
    int32_t *perm;          /* [T*K]  slots grouped by expert, ascending token within an expert */
} maple_moe_taps;

/* Human-readable name of a status code (static string). */
const char *maple_moe_status_string(int status);

/*
 * Pack int8 ternary values into the 2-bit interchange format (defined at
 * maple_moe_weights).  values: DEVICE [rows][cols] int8 in {-1,0,+1};
 * packed: DEVICE [rows][cols/16] uint32.  cols % 16 == 0.  A value outside
 * {-1,0,+1} is written as 0 and counted in *bad_count (DEVICE int32, may be
 * NULL; the caller zeroes it).
 */
int maple_moe_pack_ternary(const int8_t *values, int64_t rows, int32_t cols, uint32_t *packed,
                           int32_t *bad_count, maple_stream_t stream);

/*
 * Create a layer: validate the shape, allocate the library-owned weight copies
 * (re-laid out for the decode kernel and/or the tcgen05 GEMM, as config.flags
 * say) and a workspace for max_tokens tokens, and launch the re-layout on
 * `stream`.  *out receives the handle.  Errors: INVALID_ARG (also for unknown
 * or conflicting flags), UNSUPPORTED_SHAPE, OOM, CUDA; on error nothing stays
 * allocated.
 */
int maple_moe_create(const maple_moe_config *config, const maple_moe_weights *weights, maple_stream_t stream,
                     maple_moe_t *out);

/*
 * Routing only: topk_idx [T][K] int32 and topk_w [T][K] fp32 (rank order) and
 * expert_counts [E] int32.  x: DEVICE [T][D] bf16 (uint16 bit patterns).  Any
 * output may be NULL.  0 <= T <= max_tokens; T == 0 is a no-op.
 */
int maple_moe_route(maple_moe_t layer, const uint16_t *x, int32_t T, int32_t *topk_idx, float *topk_w,
                    int32_t *expert_counts, maple_stream_t stream);

/*
 * Full forward pass: y [T][D] fp32 from x [T][D] bf16.  taps may be NULL.
 * 0 <= T <= max_tokens; T == 0 is a no-op.
 */
int maple_moe_forward(maple_moe_t layer, const uint16_t *x, int32_t T, float *y, const maple_moe_taps *taps,
                      maple_stream_t stream);

/*
 * Layer stack with pre-norm and residual:  for l in 0..n_layers-1:
 *   x = bf16(RMSNorm(resid)) (norm weights 1, eps 1e-6);  resid = resid + layer_l(x).
 * resid: DEVICE [T][D] fp32, updated in place.  All layers must share one
 * shape.  Uses layers[0]'s workspace for x.
 */
int maple_moe_stack_forward(const maple_moe_t *layers, int32_t n_layers, float *resid, int32_t T,
                            maple_stream_t stream);

/*
 * Per-stage timing for profiling.  With events non-NULL (n_events == 4, each a
 * cudaEvent_t created by the caller on the layer's device), every later
 * maple_moe_forward on this handle records events[0] before routing,
 * events[1] after routing and the permutation, events[2] after the gate/up
 * stage and events[3] after the down/combine stage, on the call's stream.
 * events == NULL turns it off.  The handle keeps the four handles, not the
 * array.
 */
int maple_moe_set_stage_events(maple_moe_t layer, void *const *events, int32_t n_events);

/*
 * Routing without any device allocation.  The source pages have no counterpart
 * of this entry point; it exists for callers that cannot let a library call
 * cudaMalloc: processes whose device memory belongs to their own pool
 * allocator (an allocation behind the pool's back fragments it and may
 * synchronise the device) and serving loops that forbid allocation once
 * running.  No handle is needed: the router weights are read from the
 * caller's buffers and the scratch (logits, int8 codes, counters,
 * permutation) lives in a fixed 1 MiB device array inside this library, which
 * every GPU that loads the library holds until the process exits.
 * Computes exactly what maple_moe_route computes: topk_idx [T][K] int32,
 * topk_w [T][K] fp32 and expert_counts [E] int32 (may be NULL).
 * x: DEVICE [T][D] bf16; router_w: DEVICE [E][D] fp32; router_bias: DEVICE [E]
 * or NULL; all 16-byte aligned.
 * Limits (else MAPLE_ERR_INVALID_ARG / MAPLE_ERR_UNSUPPORTED_SHAPE):
 * 0 <= T <= 64, T * n_experts <= 16384, and the shape limits of
 * maple_moe_config for d_model, n_experts and top_k.
 * The first call on a device looks up the array's device address and raises
 * the routing kernel's shared-memory limit for that device; make that first
 * call before any stream capture.  Both are kept for the life of the process:
 * after a cudaDeviceReset of a device, do not call this entry point on it.  Every call uses the same array and it keeps
 * the previous call's contents (the counters that must start at zero are
 * cleared by each call on its stream), so calls whose work overlaps on the GPU
 * (other streams, other host threads) race: order them on one stream.
 * A NaN logit is ranked last; this entry point has no flag word to report it.
 */
int maple_moe_route_noalloc(const uint16_t *x, int32_t T, int32_t d_model, int32_t n_experts, int32_t top_k,
                            const float *router_w, const float *router_bias, int32_t *topk_idx, float *topk_w,
                            int32_t *expert_counts, maple_stream_t stream);

/* Read (and optionally clear) the device flag word; no synchronisation.
 * Clearing a MAPLE_FLAG_TIMEOUT here still makes the next call reset the
 * handle's internal counters (that call then returns normally). */
int maple_moe_device_flags(maple_moe_t layer, uint32_t *flags, int32_t clear);

/* maple_moe_set_debug flags (testing the failure handling only) */
#define MAPLE_DEBUG_STALL_DOWN 0x1u   /* the decode path's down kernel waits for a device word that
                                         nothing sets, so that its bounded wait expires */
#define MAPLE_DEBUG_SPLIT_SMALL 0x2u  /* decode batches of at most 8 tokens take the two-kernel expert
                                         path (gate/up kernel, down kernel, combine) instead of the
                                         fused one-kernel path (one thread-block cluster per expert) */

/*
 * Failure-handling knobs of a handle, for tests.  wait_limit_us: the limit of
 * every bounded device wait of later calls, in microseconds (0 = the default
 * 2 s; at most 60 s).  debug_flags: MAPLE_DEBUG_* bits (0 in normal use).
 * Takes effect for calls made after it returns.  Errors: INVALID_ARG.
 */
int maple_moe_set_debug(maple_moe_t layer, int32_t wait_limit_us, uint32_t debug_flags);

/* maple_moe_expert_path results */
#define MAPLE_PATH_TC 0            /* tensor-core grouped GEMMs (gate/up + SwiGLU + requantisation, down), combine */
#define MAPLE_PATH_DECODE 1        /* weight-streaming gate/up kernel, down kernel, combine kernel */
#define MAPLE_PATH_DECODE_FUSED 2  /* one kernel: a thread-block cluster per active expert, combine included */

/*
 * Which expert path a forward of T tokens takes on this handle now (its
 * configuration flags, debug flags and the device's cluster occupancy decide;
 * the routing step is the same for all).  For measurement and tests: writes
 * one of MAPLE_PATH_* to *path.  Launches nothing.  Errors: INVALID_ARG (path
 * NULL, T < 1 or above the handle's max_tokens), UNSUPPORTED_SHAPE (a
 * decode-only handle and T above its decode limit).
 */
int maple_moe_expert_path(maple_moe_t layer, int32_t T, int32_t *path);

/* Synchronise all work of the layer and free everything it owns.  NULL is a no-op. */
int maple_moe_destroy(maple_moe_t layer);

#ifdef __cplusplus
}
#endif

#endif /* MAPLE_MOE_H */
