/*
 * moe_w8a8 -- C ABI of the B200 (sm_100a) W8A8 mixture-of-experts FFN layer.
 *
 * The layer (one MoE FFN block):
 *   gate:    logits l = X W_router (+ bias), top-k experts per token with the
 *            lowest index winning ties, softmax over the k selected logits.
 *   sort:    the (token, slot) pairs grouped by expert in token order, an
 *            optional per-expert capacity dropping late arrivals.
 *   quant:   X smoothed by 1/s (SmoothQuant) and quantised to INT8 per token.
 *   experts: for each expert, INT8 x INT8 -> INT32 grouped GEMMs against
 *            per-output-channel INT8 weights; gate/up dequantised, SwiGLU,
 *            h requantised to INT8 per row; down dequantised and scaled by
 *            the routing weight.
 *   combine: the k expert outputs of each token summed in slot order.
 * Sources, by page title and section:
 *   "MiniMax-M3 W8A8 on K100AI" (mhpq.cn, MetaInfer practice notes):
 *     s1.2 W8A8 = INT8 weights x INT8 activations on the INT8 GEMM path with
 *     integer accumulation and dequantisation back to FP16/BF16; s3.2 quant
 *     config (8-bit weights per output channel, 8-bit activations per token,
 *     SmoothQuant with alpha 0.6); s4.3 keep consecutive matmuls in the INT8
 *     domain, fuse the expert FFN, pool device memory; s6.1/s6.4 smoothing
 *     and per-token quantisation against activation outliers.
 *   "Day0 adaptation of ultra-large model inference" (ruibaoantu.com),
 *     section 4, MoE operator fusion: gate, sort, grouped GEMM, un-sort and
 *     weighted sum in few kernels; top-k must equal the reference including
 *     its tie-break rule; section 2 item 2: capacity factor, dropped tokens.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device; "host" pointers are ordinary host memory.  The caller owns
 *     every buffer it passes; the library owns the prepared-weights handle
 *     until moe_w8a8_destroy.
 *   - Work is enqueued on the given stream and is asynchronous; no call
 *     synchronises the stream except moe_w8a8_prepare (which needs the
 *     smoothing statistics on the host) and moe_w8a8_check_status.
 *   - Arguments are validated before anything is enqueued; on an error the
 *     call returns a status and enqueues nothing.  No call throws or exits.
 *   - Calls that run the layer on a handle (forward, forward_host,
 *     forward_noalloc and the moe_w8a8_ep_* steps) need the handle's device
 *     to be current (the one current at prepare); otherwise they return
 *     MOE_ERR_INVALID_ARG.
 *   - Shapes: d and f multiples of 128, 1 <= top_k <= min(8, n_experts),
 *     n_experts <= 256, T >= 0 (T = 0 is a no-op).  Other shapes return
 *     MOE_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef MOE_W8A8_H
#define MOE_W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t; NULL = legacy stream */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,          /* null pointer, bad enum, alpha outside [0, 1] ...      */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,    /* see the shape rules above                             */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < moe_w8a8_workspace_size(w, T)       */
    MOE_ERR_CUDA = 4,                 /* a CUDA runtime call failed                            */
    MOE_ERR_TIMEOUT = 5,              /* a bounded device-side wait ran out (status word)      */
    MOE_ERR_OOM = 6                   /* device allocation in moe_w8a8_prepare failed          */
} moe_status;

enum { MOE_F32 = 0, MOE_BF16 = 1 };

/* Number format of the expert weights, the quantised activations and h
 * (ruibaoantu.com "Day0 adaptation" page, section 1: expert layers in INT8 or
 * FP8, activations on the same precision path as the weights).
 *   MOE_FMT_INT8: symmetric INT8, scale = amax / 127, codes rint(v / scale)
 *                 clamped to +-127; INT32 accumulation (exact).
 *   MOE_FMT_E4M3: FP8 E4M3 (finite-only OCP format, largest 448), scale =
 *                 amax / 448, codes = nearest E4M3 of v / scale (ties to even,
 *                 saturating); fp32 accumulation in the tensor cores, so the
 *                 accumulators are not reproducible bit for bit across
 *                 summation orders.  Tensor-core path only (MOE_PATH_STREAM is
 *                 refused; MOE_PATH_AUTO picks the tensor path). */
enum { MOE_FMT_INT8 = 0, MOE_FMT_E4M3 = 1 };

/* Expert GEMM path: AUTO picks STREAM for small row counts (weight-bandwidth
 * bound: each active expert's INT8 weights are read once with 128-bit loads)
 * and TENSOR otherwise (tcgen05 kind::i8 grouped GEMMs; kind::f8f6f4 for E4M3
 * experts, which always take the TENSOR path). */
enum { MOE_PATH_AUTO = 0, MOE_PATH_STREAM = 1, MOE_PATH_TENSOR = 2 };

typedef struct {
    int32_t d;                /* hidden size                                                  */
    int32_t f;                /* expert FFN intermediate size                                 */
    int32_t n_experts;        /* E                                                            */
    int32_t top_k;            /* k                                                            */
    float alpha;              /* SmoothQuant migration strength, in [0, 1] (pages use 0.6)     */
    float capacity_factor;    /* finite; <= 0: no capacity; else C = min(ceil(cf T k / E), T k) */
    int32_t renormalize;      /* 1: softmax over the k selected logits; 0: over all E          */
    int32_t in_dtype;         /* MOE_F32 or MOE_BF16: X                                       */
    int32_t out_dtype;        /* MOE_F32 or MOE_BF16: Y                                       */
    int32_t expert_format;    /* MOE_FMT_INT8 (0) or MOE_FMT_E4M3 (1)                         */
} moe_w8a8_config;

typedef struct moe_w8a8_weights moe_w8a8_weights; /* opaque, library-owned */

/* Optional intermediates for parity checks (device pointers, each may be NULL).
 * R = number of kept (token, slot) rows, at most T*k.  Rows are ordered by
 * expert, then token.  Channel order is canonical: acc1 holds gate channels
 * 0..f-1 then up channels 0..f-1. */
typedef struct {
    float* logits;       /* [T][E]  router logits incl. bias                          */
    int32_t* topk_idx;   /* [T][k]                                                    */
    float* topk_w;       /* [T][k]                                                    */
    int32_t* offsets;    /* [E+1]   first row of each expert; offsets[E] = R          */
    int32_t* row2ts;     /* [T*k]   row -> t*k + slot (first R entries valid)          */
    int32_t* ts2row;     /* [T*k]   (t, slot) -> row, -1 when dropped by capacity      */
    int8_t* xq;          /* [T][d]  INT8 smoothed activations                          */
    float* sx;           /* [T]     per-token activation scales                        */
    int32_t* acc1;       /* [T*k][2f] gate|up INT32 accumulators (first R rows)        */
    int8_t* hq;          /* [T*k][f]  INT8 h                                           */
    float* sh;           /* [T*k]     per-row h scales                                 */
    int32_t* acc2;       /* [T*k][d]  down-projection INT32 accumulators               */
    void* o;             /* [T*k][d]  weighted expert outputs (the per-slot rows the
                                          combine sums), in the output precision:
                                          bf16 for MOE_BF16 output, else fp32          */
} moe_w8a8_debug;

/*
 * Calibration statistic for SmoothQuant (mhpq.cn page s3.2: calibration
 * samples -> per-channel activation range): absmax[j] = max(absmax[j],
 * max_r |x[r][j]|) over `rows` activation rows x [rows][d] (device, dtype
 * MOE_F32 or MOE_BF16).  absmax [d] (device, fp32) is updated in place, so
 * the calibration set may come in several batches; start it at zero.
 */
moe_status moe_w8a8_calibrate_absmax(const void* x, int64_t rows, int32_t d, int32_t dtype,
                                     float* absmax, moe_stream_t stream);

/*
 * Fold SmoothQuant into the expert weights and quantise them (mhpq.cn page
 * s3.2, s6.1; formula s_j = max|X_j|^alpha / max|W_j|^(1-alpha)).
 *   w_gate, w_up  device fp32 [E][d][f]   (gate = x W_gate[e])
 *   w_down        device fp32 [E][f][d]
 *   w_router      device fp32 [d][E]      (copied; used unquantised)
 *   act_absmax    device fp32 [d]         (from moe_w8a8_calibrate_absmax)
 * max|W_j| is taken over the gate and up weights of every expert.  Gate and
 * up weights are smoothed and quantised per output channel; down weights
 * per output channel without smoothing.  The inputs may be freed afterwards.
 * Synchronises `stream` once (the O(d) scale computation runs on the host
 * in fp64).  Allocates the handle's device memory (3 d f E bytes of INT8
 * weights plus scales); returns MOE_ERR_OOM if that fails.
 */
moe_status moe_w8a8_prepare(const moe_w8a8_config* cfg, const float* w_gate, const float* w_up,
                            const float* w_down, const float* w_router, const float* act_absmax,
                            moe_stream_t stream, moe_w8a8_weights** out);

/* Bytes of device workspace moe_w8a8_forward needs for up to max_tokens
 * tokens (0 on a NULL handle or negative max_tokens). */
size_t moe_w8a8_workspace_size(const moe_w8a8_weights* w, int32_t max_tokens);

/*
 * Run the layer on T tokens.
 *   x              device [T][d], cfg.in_dtype, 16-byte aligned
 *   router_bias    device fp32 [E] added to every token's logits, or NULL;
 *                  16-byte aligned
 *   router_logits  device fp32 [T][E] used instead of X W_router, or NULL;
 *                  16-byte aligned
 *   y              device [T][d], cfg.out_dtype, 16-byte aligned
 *   workspace      device, >= moe_w8a8_workspace_size(w, T) bytes, 256-byte aligned
 * The kernels read and write x, y, router_bias and router_logits with
 * 16-byte vector accesses: a NULL or misaligned pointer (NULL is allowed for
 * the two optional ones) returns MOE_ERR_INVALID_ARG before the handle is
 * read and before anything is enqueued.  The buffers must hold the sizes
 * above; the library cannot check that (the Python binding does).
 *   dbg            NULL, or device pointers receiving intermediates
 * Allocates nothing; all scratch lives in the caller's workspace.  Calls
 * that share a workspace must not overlap on the device.
 * With few rows per expert (T*k <= 512 on the tensor path) the expert FFN
 * runs as one persistent launch whose thread blocks wait on one another's
 * results; tiles are taken from a device-wide counter in dependency order,
 * so every wait is on work a running block already holds and the launch
 * progresses even when other streams keep some of its blocks off the SMs.
 * All such waits are bounded (2 s) and report MOE_ERR_TIMEOUT
 * (moe_w8a8_check_status) instead of hanging.
 * A handle from moe_w8a8_prepare_shard that does not hold every expert
 * returns MOE_ERR_INVALID_ARG (here, in moe_w8a8_forward_host and in
 * moe_w8a8_forward_noalloc): it runs through the moe_w8a8_ep_* calls.
 */
moe_status moe_w8a8_forward(const moe_w8a8_weights* w, const void* x, int32_t T,
                            const float* router_bias, const float* router_logits, void* y,
                            void* workspace, size_t workspace_bytes, const moe_w8a8_debug* dbg,
                            moe_stream_t stream);

/*
 * moe_w8a8_forward from host memory: copies x (and router_logits /
 * router_bias when given) host -> device into the workspace, runs the
 * layer, and copies y device -> host, all enqueued on `stream`.  Host
 * buffers should be page-locked for the copies to be asynchronous; y is
 * valid once the stream has been synchronised.
 */
moe_status moe_w8a8_forward_host(const moe_w8a8_weights* w, const void* x_host, int32_t T,
                                 const float* router_bias_host, const float* router_logits_host,
                                 void* y_host, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream);

/*
 * moe_w8a8_forward for callers that cannot allocate device memory.
 *
 * No counterpart on the pages: this entry point exists for library users,
 * not for the method.  Some callers may not call cudaMalloc at all on their
 * request path: a serving process that plans every device byte at start-up
 * and forbids allocation afterwards, or a plugin hosted by a framework that
 * owns the device allocator and gives the plugin no allocation hook.  Such a
 * caller passes only its inputs and outputs; the scratch memory comes from a
 * fixed array compiled into this library (MOE_NOALLOC_SCRATCH_BYTES bytes of
 * device memory, held on every GPU that loads the library until the process
 * exits).  Nothing is allocated by this call: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 *   x, router_bias, router_logits, y: as for moe_w8a8_forward (device).
 * T is limited by the array: a call whose moe_w8a8_workspace_size(w, T)
 * exceeds MOE_NOALLOC_SCRATCH_BYTES returns MOE_ERR_WORKSPACE_TOO_SMALL and
 * enqueues nothing (for the d=4096, E=64, top-4, f=1536 decode layer that is
 * T up to 82 tokens).
 * The first call on a device looks up the array's device address with that
 * device current (cudaGetSymbolAddress) and caches it; make that first call
 * before any stream capture.  Every call on a device shares the one array,
 * which keeps the previous call's contents (the forward writes every scratch
 * word it later reads, so nothing needs clearing); calls that overlap on the
 * GPU (different streams, or different threads) race on it and must be
 * serialised by the caller.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (8u << 20)
moe_status moe_w8a8_forward_noalloc(const moe_w8a8_weights* w, const void* x, int32_t T,
                                    const float* router_bias, const float* router_logits,
                                    void* y, moe_stream_t stream);

/*
 * Measurement aid (no counterpart on the pages): the dense 8-bit tensor-core
 * rate this library's own MMA reaches on the current device, the denominator
 * of the tensor-bound roofline.  Enqueues one launch of one thread block per
 * SM; each issues mma_per_sm tcgen05 MMAs of M=128 x N=256 x K=32 (kind::i8
 * for MOE_FMT_INT8, kind::f8f6f4 E4M3 for MOE_FMT_E4M3) back to back on
 * operands held in shared memory (pseudo-random codes), with no data
 * movement.  *ops_out receives the launch's operation count (2 x M x N x K x
 * MMAs x SMs); the caller times the launch (events on `stream`).
 * 0 < mma_per_sm <= MOE_PEAK_MAX_MMA (about a second of work), else
 * MOE_ERR_INVALID_ARG.  Allocates nothing.
 */
#define MOE_PEAK_MAX_MMA (1LL << 24)
moe_status moe_w8a8_tensor_peak_loop(int32_t expert_format, int64_t mma_per_sm, double* ops_out,
                                     moe_stream_t stream);

/* Select the expert GEMM path (MOE_PATH_*). */
moe_status moe_w8a8_set_path(moe_w8a8_weights* w, int32_t path);

/* Row count at or below which MOE_PATH_AUTO uses the streaming path. */
moe_status moe_w8a8_set_stream_threshold(moe_w8a8_weights* w, int32_t max_rows);

/*
 * Row count (T * k) at or below which the tensor-core path runs GEMM1, the
 * requantisation of h and GEMM2 as one persistent launch with per-expert
 * dependencies between its thread blocks (above it: three launches).  The
 * results are identical either way; max_rows >= 0.  Changing it can change
 * moe_w8a8_workspace_size (the fused launch keeps a few counters per 128-row
 * tile in the workspace).
 */
moe_status moe_w8a8_set_fused_threshold(moe_w8a8_weights* w, int64_t max_rows);

/*
 * Whether the tensor-core path's separate GEMM launches run on pairs of SMs:
 * a cluster of two thread blocks computes 256-row tiles with one
 * tcgen05.mma.cta_group::2 per K slice, each SM loading half of the tile's
 * weight columns (less operand traffic per MMA, deeper pipelines) at the cost
 * of MMA work on the unused rows of each expert's last 256-row tile.
 * mode 0: never; 1: always; 2 (default): when T * k >= 256 * E, i.e. the rows
 * per expert fill such tiles on average.  The results are identical.
 */
moe_status moe_w8a8_set_cta_pairs(moe_w8a8_weights* w, int32_t mode);

/*
 * Saturating activation clip (mhpq.cn page s6.4, the third defence against
 * activation outliers: cut values at a threshold instead of stretching the
 * scale to the maximum; gtnt.cn page s3.2: the threshold is a percentile of
 * the calibration activations, 99.9 there).  With clip > 0 every forward
 * quantises token t of the smoothed input x' = x * inv_s with the range
 * a_t = min(max_j |x'_tj|, clip): scale a_t / 127, codes rint(x' / scale)
 * clamped to +-127, so values beyond the clip saturate.  clip = 0 turns it
 * off (the default).  Only the layer input is clipped, not the expert's
 * intermediate h.  Returns MOE_ERR_INVALID_ARG for a negative or non-finite
 * clip.  Takes effect from the next forward; do not change it while a
 * forward on this handle may be in flight.
 */
moe_status moe_w8a8_set_act_clip(moe_w8a8_weights* w, float clip);

/*
 * The clip threshold from calibration rows x [rows][d] (device, dtype
 * MOE_F32 or MOE_BF16): the nearest-rank `percent` percentile (0 < percent
 * <= 100) of |x[r][j] * inv_s[j]| over every element, i.e. the
 * ceil(percent/100 * rows * d)-th smallest, written to *clip_host.  Calibration
 * helper, not part of the forward: it allocates rows * d * 4 bytes of device
 * memory, runs one kernel, copies the values to the host and selects there,
 * and synchronises `stream`.  Does not change the handle; pass the value to
 * moe_w8a8_set_act_clip.
 */
moe_status moe_w8a8_calibrate_act_clip(const moe_w8a8_weights* w, const void* x, int64_t rows,
                                       int32_t dtype, double percent, float* clip_host,
                                       moe_stream_t stream);

/* Smoothing scales s [d] copied to host memory. */
moe_status moe_w8a8_get_smooth_scales(const moe_w8a8_weights* w, float* s_host);

/*
 * Copy the prepared weights out in canonical layout (device pointers, each
 * may be NULL): wq_gate, wq_up INT8 [E][f][d]; sw_gate, sw_up fp32 [E][f];
 * wq_down INT8 [E][d][f]; sw_down fp32 [E][d]; inv_s fp32 [d].
 */
moe_status moe_w8a8_export_weights(const moe_w8a8_weights* w, int8_t* wq_gate, int8_t* wq_up,
                                   float* sw_gate, float* sw_up, int8_t* wq_down, float* sw_down,
                                   float* inv_s, moe_stream_t stream);

/*
 * Synchronise `stream` and read the handle's device status word: MOE_OK,
 * MOE_ERR_TIMEOUT when a bounded wait in a kernel ran out since the last
 * check, MOE_ERR_INVALID_ARG when moe_w8a8_ep_experts received a row for an
 * expert this handle does not hold (the word is then cleared), or
 * MOE_ERR_CUDA on a pending CUDA error.
 */
moe_status moe_w8a8_check_status(const moe_w8a8_weights* w, moe_stream_t stream);

/*
 * Diagnostics after MOE_ERR_TIMEOUT: synchronise `stream` and copy the
 * handle's status words to words_host[0..n) (n <= 16): word 0 is the status
 * code, words 1-4 say where the first bounded wait gave up: word 1 the site,
 * word 2 the thread block, words 3-4 site-specific.  Sites of the tensor-core
 * expert kernels: 1 producer waiting for a free stage, 2 MMA issuer waiting
 * for a free accumulator, 3 MMA issuer waiting for a full stage, 4 epilogue
 * waiting for a full accumulator (words 3-4: tile, awaited phase parity);
 * of the fused expert launch also 6 a down-projection producer waiting for
 * an m-tile's h codes (words 3-4: tile, m-tile), 7 a requantisation warp
 * waiting for an m-tile's h to be complete (word 3: m-tile), 8-10 the producer, MMA issuer and
 * epilogue waiting on the block's tile ring, 16 a down-projection epilogue
 * waiting for an m-tile's h scales (words 3-4: tile, m-tile); 11-13 the certified router's
 * producer, MMA issuer and epilogue.  Site 14 (with MOE_ERR_INVALID_ARG): a
 * received expert-parallel row names an expert outside the handle's range
 * (words 2-3: row index, expert); site 15 (with MOE_ERR_INVALID_ARG): a
 * received fixed block's row count is outside [0, block rows - 1] (words 2-3:
 * block, count); site 17 (with MOE_ERR_INVALID_ARG): the fused expert launch's
 * plan for at most 32 tokens met an m-tile of more than 32 rows (words 3-4:
 * m-tile, rows; an internal consistency check).  Does not clear them.
 */
moe_status moe_w8a8_status_words(const moe_w8a8_weights* w, int32_t* words_host, int32_t n,
                                 moe_stream_t stream);

/*
 * Bound on each wait of one thread block for results of another block (the
 * fused expert launch: a down-projection tile waiting for its rows' h codes,
 * a requantisation warp waiting for a finished m-tile), in nanoseconds, from
 * 1 ms to 60 s; default 2 s.  When such a wait runs out the launch records
 * MOE_ERR_TIMEOUT and the place (moe_w8a8_status_words), every block of it
 * stops issuing work, waits (bounded) for its copies and MMAs in flight,
 * frees its tensor memory and returns, so the GPU context stays usable;
 * moe_w8a8_check_status reports it.  Waits on a block's own copies and MMAs
 * keep a fixed 2 s bound.  (No counterpart on the pages, whose watchdog is a
 * host-side check; "One night of MoE inference optimisation", s6.4.)
 */
moe_status moe_w8a8_set_wait_budget(moe_w8a8_weights* w, int64_t ns);

/*
 * Testing aid for the failure path above, off by default: with m_tile >= 0
 * every later fused expert launch of this handle computes as usual but never
 * releases the h codes of that 128-row tile (one expert's rows), so the
 * down-projection tiles that need them wait until the budget runs out and the
 * launch ends with MOE_ERR_TIMEOUT; the output of such a call is undefined.
 * m_tile = -1 turns it off.  Launches that are not the fused one ignore it.
 */
moe_status moe_w8a8_test_withhold_release(moe_w8a8_weights* w, int32_t m_tile);

/* Free the handle and its device memory (NULL is a no-op).  The caller makes
 * sure no enqueued forward still uses it. */
void moe_w8a8_destroy(moe_w8a8_weights* w);

/* Static description of a status code. */
const char* moe_status_string(moe_status s);

/* Number of kernels the last successful forward on this handle enqueued. */
int32_t moe_w8a8_last_launch_count(const moe_w8a8_weights* w);


/* Stages of one forward, for per-stage timing. */
enum {
    MOE_STAGE_ROUTER = 0,   /* router logits X W_router (skipped when logits are given) */
    MOE_STAGE_TOPK = 1,     /* top-k + gate softmax                                     */
    MOE_STAGE_PERMUTE = 2,  /* histogram + stable scatter by expert                     */
    MOE_STAGE_QUANT = 3,    /* smoothing + per-token INT8 quantisation                  */
    MOE_STAGE_GEMM1 = 4,    /* gate/up grouped GEMM                                     */
    MOE_STAGE_REQUANT = 5,  /* SwiGLU + per-row INT8 requantisation (when not fused)    */
    MOE_STAGE_GEMM2 = 6,    /* down grouped GEMM + dequant x routing weight             */
    MOE_STAGE_COMBINE = 7,  /* un-sort + weighted sum                                   */
    MOE_N_STAGES = 8
};

/*
 * Measurement aid: from now on, record a CUDA event pair around every stage
 * of the next max_forwards forwards on this handle, on the forward's stream
 * (a stage that does not run records an empty interval).  Allocates the
 * events here, never inside a forward.
 */
moe_status moe_w8a8_profile_start(moe_w8a8_weights* w, int32_t max_forwards);

/*
 * As moe_w8a8_profile_start, but only the stages whose bit (1 << stage) is set
 * in stage_mask record their event pair; the others record nothing and read
 * back as 0 ms.  Bracketing one stage alone leaves every other boundary of the
 * forward free of events, so the launches run as in a plain forward except at
 * that stage's own two boundaries.
 * stage_mask == 0 or with bits at or above MOE_N_STAGES: MOE_ERR_INVALID_ARG.
 */
moe_status moe_w8a8_profile_start_stages(moe_w8a8_weights* w, int32_t max_forwards, uint32_t stage_mask);

/* Synchronise the recorded events and write ms_host[i * MOE_N_STAGES + s],
 * the time of stage s in recorded forward i, for up to `capacity` forwards.
 * Returns the number of forwards written (negative on a CUDA error).
 * Stages left out by the mask read 0. */
int32_t moe_w8a8_profile_read(moe_w8a8_weights* w, float* ms_host, int32_t capacity);

/* Stop recording and free the events. */
moe_status moe_w8a8_profile_stop(moe_w8a8_weights* w);

/* Static name of a stage ("router", "topk", ...), or "?" . */
const char* moe_w8a8_stage_name(int32_t stage);

/* ------------------------------------------------------------------------
 * Expert parallelism.  "Day0 adaptation of ultra-large model inference",
 * section 3: the experts are spread over the GPUs and each layer moves its
 * tokens with one All-to-All each way; section 4: the operator chain gate ->
 * sort -> All-to-All -> grouped GEMM -> reverse All-to-All -> un-sort ->
 * weighted sum.
 *
 * G ranks hold G contiguous ranges of the layer's E experts (rank g: experts
 * [g E / G, (g + 1) E / G) when G divides E; any contiguous split works).
 * Each rank routes and quantises its own T tokens against all E experts; the
 * result on every rank equals moe_w8a8_forward on that rank's tokens with a
 * handle holding all experts (the same capacity rule, applied to those T
 * tokens).  One layer on one rank:
 *   1. moe_w8a8_ep_dispatch: router, top-k, sort and quantisation.  Writes
 *      the kept (token, slot) rows, expert-major and in token order within
 *      an expert (so the rows for one rank are contiguous), to `send`, and
 *      the per-expert row offsets [E + 1] to expert_offsets.
 *   2. the caller exchanges, per destination rank, the rows of its experts
 *      (one All-to-All of whole rows; row counts from expert_offsets).
 *   3. moe_w8a8_ep_experts on the received rows (in any order): the local
 *      experts' grouped GEMMs; writes the fp32 output row of each received
 *      row, in the received order.
 *   4. the caller returns the output rows to their senders (the reverse
 *      All-to-All: every row goes back to the rank and position it came from).
 *   5. moe_w8a8_ep_combine: each token's output as the sum of its kept slots
 *      in slot order, from the returned rows in the order of `send`.
 * Row layout (moe_w8a8_ep_row_bytes(w) = d + 16 bytes per row): the d INT8
 * (or E4M3) codes of the token, then fp32 activation scale, fp32 gate weight,
 * int32 global expert, int32 t * k + slot on the sending rank.
 * ------------------------------------------------------------------------ */

/* Bytes per dispatched row: d + 16 (0 on a NULL handle). */
int32_t moe_w8a8_ep_row_bytes(const moe_w8a8_weights* w);

/*
 * aw[j] = max over the given n_local experts e and every output n of
 * |w_gate[e][j][n]| and |w_up[e][j][n]|: the weight statistic of the
 * SmoothQuant scale ("MiniMax-M3 W8A8 on K100AI" s6.1/s6.4).  The layer's aw
 * is the maximum over all ranks (an all-reduce with MAX of this per-rank
 * value), which every rank then passes to moe_w8a8_prepare_shard.
 *   w_gate, w_up  device fp32 [n_local][d][f];  aw  device fp32 [d]
 * Asynchronous on `stream`.
 */
moe_status moe_w8a8_gateup_absmax(const moe_w8a8_config* cfg, int32_t n_local, const float* w_gate,
                                  const float* w_up, float* aw, moe_stream_t stream);

/*
 * moe_w8a8_prepare for experts [expert_first, expert_first + n_local) of the
 * layer `cfg` (cfg.n_experts = all E experts).
 *   w_gate, w_up   device fp32 [n_local][d][f] (those experts only)
 *   w_down         device fp32 [n_local][f][d]
 *   w_router       device fp32 [d][E] (the whole router)
 *   act_absmax     device fp32 [d]
 *   gateup_absmax  device fp32 [d], the layer's aw over ALL E experts (see
 *                  moe_w8a8_gateup_absmax), so that every rank computes the
 *                  same smoothing s and quantises its tokens identically
 * Returns MOE_ERR_INVALID_ARG for a range outside [0, E) or a NULL pointer;
 * otherwise as moe_w8a8_prepare.  The handle serves moe_w8a8_ep_* only
 * (unless it holds all E experts).
 */
moe_status moe_w8a8_prepare_shard(const moe_w8a8_config* cfg, int32_t expert_first, int32_t n_local,
                                  const float* w_gate, const float* w_up, const float* w_down,
                                  const float* w_router, const float* act_absmax, const float* gateup_absmax,
                                  moe_stream_t stream, moe_w8a8_weights** out);

/* Workspace of moe_w8a8_ep_dispatch and moe_w8a8_ep_combine for up to
 * max_tokens tokens; of moe_w8a8_ep_experts for `rows` received rows. */
size_t moe_w8a8_ep_dispatch_workspace_size(const moe_w8a8_weights* w, int32_t max_tokens);
size_t moe_w8a8_ep_experts_workspace_size(const moe_w8a8_weights* w, int32_t rows);

/*
 * Step 1 of the expert-parallel layer on this rank's T tokens.
 *   x, router_bias, router_logits   as in moe_w8a8_forward
 *   send            device [T * k][moe_w8a8_ep_row_bytes(w)] bytes, 16-byte
 *                   aligned; rows [0, R) are written, R = expert_offsets[E]
 *   expert_offsets  device int32 [E + 1]: the rows of expert e are
 *                   [expert_offsets[e], expert_offsets[e + 1]) (zeros for T = 0)
 *   workspace       device, >= moe_w8a8_ep_dispatch_workspace_size(w, T),
 *                   256-byte aligned; it keeps the token -> row map that
 *                   moe_w8a8_ep_combine reads, so it must not be reused in
 *                   between
 *   dbg             NULL, or routing intermediates (logits, topk_idx, topk_w,
 *                   offsets, row2ts, ts2row, xq, sx)
 */
moe_status moe_w8a8_ep_dispatch(const moe_w8a8_weights* w, const void* x, int32_t T, const float* router_bias,
                                const float* router_logits, void* send, int32_t* expert_offsets, void* workspace,
                                size_t workspace_bytes, const moe_w8a8_debug* dbg, moe_stream_t stream);

/*
 * Step 3: the experts this handle holds, on R received rows.
 *   recv      device [R][moe_w8a8_ep_row_bytes(w)] bytes, 16-byte aligned,
 *             rows as written by moe_w8a8_ep_dispatch on any rank of the
 *             same layer, each naming one of this handle's experts
 *   o_rows    device fp32 [R][d], 16-byte aligned: o_rows[r] = the routing
 *             weight x the expert's output for received row r
 *   workspace device, >= moe_w8a8_ep_experts_workspace_size(w, R), 256-byte aligned
 *   dbg       NULL, or the expert side's intermediates by local sorted row
 *             (topk_idx = local expert per received row, offsets [n_local + 1],
 *             row2ts / ts2row between received and sorted rows, sx, acc1,
 *             hq, sh, acc2, o)
 * A row naming an expert outside this handle's range is reported through
 * the status word (moe_w8a8_check_status: MOE_ERR_INVALID_ARG) and its
 * output is meaningless.  R = 0 is a no-op.
 */
moe_status moe_w8a8_ep_experts(const moe_w8a8_weights* w, const void* recv, int32_t R, float* o_rows,
                               void* workspace, size_t workspace_bytes, const moe_w8a8_debug* dbg,
                               moe_stream_t stream);

/*
 * Step 5: y [T][d] (cfg.out_dtype, device, 16-byte aligned) from the returned
 * rows o_rows (device fp32 [R][d], in the row order of `send`, 16-byte
 * aligned and never NULL, also when R = 0: pass any valid device address
 * then, it is not read) and the workspace of the matching
 * moe_w8a8_ep_dispatch with the same T.  A NULL or misaligned pointer returns
 * MOE_ERR_INVALID_ARG before anything is enqueued.
 */
moe_status moe_w8a8_ep_combine(const moe_w8a8_weights* w, const float* o_rows, int32_t T, void* y,
                               const void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * The same layer with a fixed-block exchange, for decode-sized batches: no
 * row count ever has to reach the host.  ("Day0 adaptation of ultra-large
 * model inference", section 3: one All-to-All each way; here both have sizes
 * known in advance.)  Every rank uses the same block_tokens B >= its T.  Rank
 * g's block for peer h is moe_w8a8_ep_block_rows(w, B) = B k + 1 rows of
 * moe_w8a8_ep_row_bytes(w) bytes: a header row, whose first int32 is the
 * number n of rows for h's experts (the rest of the header zero), then those
 * n rows in the order of `send`; rows past n are unused and may hold
 * anything.  One layer on one rank of G:
 *   1. moe_w8a8_ep_dispatch as above;
 *   2. moe_w8a8_ep_pack: `send` into G blocks, one per destination;
 *   3. an All-to-All of equal parts (one block each way per peer);
 *   4. moe_w8a8_ep_experts_blocked on the G received blocks: the output row
 *      of every received row at the same position of the output blocks
 *      (fp32, d per row; headers and unused rows get zeros);
 *   5. an All-to-All of equal parts back (one output block per peer);
 *   6. moe_w8a8_ep_combine_blocked: each token's output from the returned
 *      blocks (the position of each kept slot follows from the dispatch's
 *      row offsets, kept in its workspace).
 * rank_first: host int32 [G + 1], rank g holding experts
 * [rank_first[g], rank_first[g + 1]): rank_first[0] = 0, strictly increasing,
 * rank_first[G] = E; G from 1 to 64.
 * ------------------------------------------------------------------------ */

/* Rows per block, B k + 1 (0 on a NULL handle or B < 1). */
int32_t moe_w8a8_ep_block_rows(const moe_w8a8_weights* w, int32_t block_tokens);

/*
 * Step 2: blocks, device [G][moe_w8a8_ep_block_rows(w, B)][row bytes],
 * 16-byte aligned, from `send` and the expert_offsets (device) of the
 * preceding moe_w8a8_ep_dispatch (whose T must be <= B).  A count above the
 * block's capacity cannot occur when T <= B; the receiving side reports one
 * (status word site 15) and reads it as 0.  MOE_ERR_INVALID_ARG for a NULL or
 * misaligned pointer or bad rank_first.
 */
moe_status moe_w8a8_ep_pack(const moe_w8a8_weights* w, const void* send, const int32_t* expert_offsets,
                            const int32_t* rank_first, int32_t world, int32_t block_tokens, void* blocks,
                            moe_stream_t stream);

/* Workspace of moe_w8a8_ep_experts_blocked for G blocks of B tokens. */
size_t moe_w8a8_ep_experts_blocked_workspace_size(const moe_w8a8_weights* w, int32_t world,
                                                  int32_t block_tokens);

/*
 * Step 4: the experts this handle holds, on the G received blocks (device,
 * 16-byte aligned, as written by moe_w8a8_ep_pack on the G ranks in rank
 * order).  o_blocks: device fp32 [G][block rows][d], 16-byte aligned; the
 * output row of received row i of block g at row i of output block g.  The
 * row counts are read on the device.  Errors and dbg as moe_w8a8_ep_experts,
 * with R = G x block rows and each header and unused row left out.
 */
moe_status moe_w8a8_ep_experts_blocked(const moe_w8a8_weights* w, const void* blocks, int32_t world,
                                       int32_t block_tokens, float* o_blocks, void* workspace,
                                       size_t workspace_bytes, const moe_w8a8_debug* dbg, moe_stream_t stream);

/*
 * Step 6: y [T][d] (cfg.out_dtype, device, 16-byte aligned) from the G
 * returned output blocks (device fp32 [G][block rows][d], 16-byte aligned:
 * block g from rank g) and the workspace of the matching moe_w8a8_ep_dispatch
 * with the same T (T <= B).  MOE_ERR_INVALID_ARG for a NULL or misaligned
 * pointer or bad rank_first, before anything is enqueued.
 */
moe_status moe_w8a8_ep_combine_blocked(const moe_w8a8_weights* w, const float* o_blocks, int32_t T,
                                       const int32_t* rank_first, int32_t world, int32_t block_tokens, void* y,
                                       const void* workspace, size_t workspace_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_W8A8_H */
