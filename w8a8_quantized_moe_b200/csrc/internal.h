// Internal declarations of the W8A8 MoE library: the prepared-weights handle,
// the workspace layout and the kernel launchers (one per .cu file group).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_w8a8.h"

struct moe_w8a8_weights {
    moe_w8a8_config cfg;
    int device;
    int num_sms;
    int path;               // MOE_PATH_*
    int stream_max_rows;    // AUTO: streaming path when T*k <= this
    float act_clip;         // > 0: cap of each token's smoothed range (saturating clip)
    // experts held: global experts [ep_first, ep_first + n_local) of the layer's
    // cfg.n_experts (all of them unless prepared as an expert-parallel shard)
    int ep_first;
    int n_local;
    int last_launches;
    // prepared weights (device)
    int8_t* w_gu;     // [n_local][2f][d]: per 128-channel block, 128 gate rows then 128 up rows
    // The same INT8 (or E4M3) weights for the separate GEMM launches, tiled:
    // the 256-row x 128-byte box that one k-block of a tile loads is 32 KB of
    // contiguous memory ([row tile][k-block][256 rows][128 bytes]).  Measured
    // on one box: large layer 3.05 -> 2.94 ms (its HBM-bound GEMM1 1.63 -> 1.55
    // ms), while the fused decode launch was 2-3% faster on the canonical
    // layout (many CTAs each reading 128 bytes of 256 rows spread the requests
    // over more DRAM channels), so it keeps that one.
    int8_t* w_gu_t;
    int8_t* w_dn_t;
    int8_t* w_dn;     // [n_local][d][f]
    float* sw_gate;   // [n_local][f]
    float* sw_up;     // [n_local][f]
    float* sw_dn;     // [n_local][d]
    float* inv_s;     // [d]
    float* w_router;  // [d][E]
    // certified tensor-core router (bf16 X): W_g split into bf16 hi + lo rows
    // [rt_epad][d] (experts padded with zero rows), W_g transposed [E][d] fp32
    // for the exact re-evaluation, and max_e |W_g[j][e]| [d]; the last two
    // lane-interleaved (channel 32 i + p at [i / 4][p][i % 4])
    uint16_t* rt_hi;
    uint16_t* rt_lo;
    float* rt_wt;
    float* rt_wmax;
    int rt_epad;      // 0: no tensor-core router for this handle
    float* s_host;    // [d] (host)
    int32_t* status;  // device status word
    uint64_t wait_budget_ns;   // bound on a block's wait for another block's results
    int test_skip_ready;       // testing aid: fused launch withholds this m-tile's ready flag (-1: none)
    int64_t fused_max_rows;    // tensor path: T*k at or below which GEMM1, requant and GEMM2 are one launch
    // tensor maps of the weights for the tensor-core path (built at prepare):
    // canonical layout (the fused launch), the tiled copies (the separate GEMM
    // launches), and the tiled copies in 128-row boxes (one CTA of a pair loads
    // half a tile)
    CUtensorMap tm_w_gu;
    CUtensorMap tm_w_dn;
    CUtensorMap tm_w_gu_t, tm_w_dn_t, tm_w_gu_t_half, tm_w_dn_t_half;
    int cta_pairs;             // separate GEMM launches on SM pairs: 0 never, 1 always, 2 by rows per expert
    bool tmaps_ok;
    CUtensorMap tm_rt_hi;
    CUtensorMap tm_rt_lo;
    // per-stage event timing (measurement aid)
    cudaEvent_t* prof_events;   // [prof_max][MOE_N_STAGES][2]
    int prof_max;
    int prof_n;
    uint32_t prof_mask;         // stages that record their event pair
};

namespace moe {

constexpr int kGuBlock = 128;       // gate/up interleave block (channels)
constexpr int kPermChunk = 2048;    // (t, slot) entries per permute block
constexpr int kMaxK = 8;
constexpr int kMaxE = 256;

// Byte offsets of the forward workspace for T tokens.
struct WsLayout {
    size_t x_stage, y_stage, logits_stage, bias_stage;   // forward_host staging
    size_t logits, topk_idx, topk_w;
    size_t logits_sel;           // certified router: exact-or--inf logits [T][E]
    size_t hist, offsets, meta, active, tiles, pairs;
    size_t row2ts, ts2row;
    size_t xq, sx, aq;
    size_t acc1, hq, sh, o;
    size_t h32, pamax;           // tensor path: fp32 h, per-row partial maxima
    size_t fused_sync;           // fused tensor launch: its counters and queue (cleared per forward)
    int fused_words;             // their number (0: no fused launch)
    size_t total;
};
// Which calls use the layout: the whole forward; the routing side of the
// expert-parallel layer (dispatch and combine: routing state, token codes,
// no expert buffers); or its expert side (received rows, no routing).
enum WsPart { WS_FORWARD, WS_ROUTE, WS_EXPERTS };
WsLayout ws_layout(const moe_w8a8_weights* w, int T, WsPart part = WS_FORWARD);

// Expert-parallel row: d code bytes, then this trailer.
struct EpTrailer {
    float sx;        // the token's activation scale
    float w;         // the slot's gate weight
    int32_t expert;  // global expert
    int32_t ts;      // t * k + slot on the sending rank
};
constexpr int kEpTrailerBytes = 16;
static_assert(sizeof(EpTrailer) == kEpTrailerBytes, "trailer layout");

// meta[] words written by the permute scatter kernel
enum { META_R = 0, META_NACTIVE = 1, META_NTILES = 2, META_NPAIRS = 3, META_WORDS = 8 };
constexpr int kTileM = 128;   // rows per tensor-core tile
constexpr int kPairM = 256;   // rows per tile of a CTA pair (two SMs, one 256-row MMA)

// ------------------------------------------------------------------ kernels
cudaError_t launch_calib_absmax(const void* x, int64_t rows, int d, int dtype, float* absmax,
                                cudaStream_t s);
cudaError_t launch_gateup_input_absmax(const float* w_gate, const float* w_up, int E, int d, int f,
                                       float* aw, cudaStream_t s);
// Quantise column-major channels: W [E][K][N] fp32 (input j, output n), optional
// per-input smoothing s[K]; channel n goes to out row map(n) of [E][rows][K].
// fmt: MOE_FMT_INT8 or MOE_FMT_E4M3 (codes stored as bytes either way)
cudaError_t launch_quantize_channels(const float* w, const float* smooth, int E, int K, int N,
                                     int8_t* out, int out_rows, int row_block, int row_stride,
                                     int row_base, float* sw, int fmt, cudaStream_t s);
cudaError_t launch_export_gateup(const int8_t* w_gu, int E, int d, int f, int8_t* gate,
                                 int8_t* up, cudaStream_t s);

cudaError_t launch_router_logits(const void* x, int in_dtype, const float* wr, int T, int d, int E,
                                 float* logits, cudaStream_t s);
cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, int renorm,
                        int32_t* idx, float* wts, float* logits_out, cudaStream_t s);
// zero_words[0, n_zero): counters a later kernel of the forward starts from
// zero (the fused expert launch); block 0 of the scatter clears them.
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int cap, int32_t* hist,
                           int32_t* offsets, int32_t* row2ts, int32_t* ts2row, int32_t* meta,
                           int32_t* active, int32_t* tiles, int32_t* pairs, cudaStream_t s,
                           int32_t* zero_words = nullptr, int n_zero = 0);
bool route_small_ok(int T, int k);
cudaError_t launch_route_small(const float* logits, const float* bias, int T, int E, int k,
                               int renorm, int cap, int32_t* idx, float* wts, float* logits_out,
                               int32_t* offsets, int32_t* row2ts, int32_t* ts2row, int32_t* meta,
                               int32_t* active, int32_t* tiles, int32_t* pairs, int32_t* zero_words, int n_zero,
                               cudaStream_t s);
// act_clip > 0 caps each token's range (saturating clip), 0 = off.  Codes of
// each kept (t, slot) go to row ts2row of aq (row stride aq_ld bytes; aq may be
// null); with wts and idx given, an EpTrailer follows the d codes of each row.
cudaError_t launch_smooth_quant(const void* x, int in_dtype, const float* inv_s, float act_clip, int T,
                                int d, int k, const int32_t* ts2row, int8_t* xq, float* sx, int8_t* aq,
                                int64_t aq_ld, const float* wts, const int32_t* idx, int fmt, cudaStream_t s);
// Expert-parallel receive side.  Local expert of each received row (its
// trailer's expert - ep_first); an expert outside [0, n_local) is recorded in
// status (MOE_ERR_INVALID_ARG, site kSiteEpExpert) and the row runs through
// local expert 0.  With block_rows > 0 the rows are fixed blocks of that many
// rows, each a header row (row count) and then the rows: headers and rows past
// the count get idx -1 (left out); a count outside [0, block_rows - 1] is
// recorded (site kSiteEpBlock) and read as 0.
constexpr int kSiteEpExpert = 14;
constexpr int kSiteEpBlock = 15;

cudaError_t launch_ep_read_experts(const uint8_t* recv, int R, int64_t row_bytes, int d, int block_rows,
                                   int ep_first, int n_local, int32_t* idx, int32_t* status, cudaStream_t s);

// The expert ranges of the ranks of a fixed-block exchange: rank g holds
// global experts [first[g], first[g + 1]).
constexpr int kEpMaxWorld = 64;
struct EpRanks {
    int32_t first[kEpMaxWorld + 1];
};
// Send rows (expert-major, `offsets` the E + 1 row offsets) into world fixed
// blocks of block_rows rows: header row with the count, then the rows.
cudaError_t launch_ep_pack(const uint8_t* send, const int32_t* offsets, const EpRanks& ranks, int world,
                           int block_rows, int64_t row_bytes, uint8_t* blocks, cudaStream_t s);
// Codes of received row r to row ts2row[r] of dst (row r when ts2row is
// null; nothing when ts2row[r] < 0), its scale and gate weight to sx[r] and
// wts[r].
cudaError_t launch_ep_gather(const uint8_t* recv, int R, int64_t row_bytes, int d, const int32_t* ts2row,
                             int8_t* dst, float* sx, float* wts, cudaStream_t s);
// out[r][j] = |fp32(x[r][j] * inv_s[j])| (calibration of the activation clip)
cudaError_t launch_scaled_abs(const void* x, int64_t rows, int d, int dtype, const float* inv_s, float* out,
                              cudaStream_t s);

cudaError_t launch_stream_gateup(const moe_w8a8_weights* w, int T, const int8_t* xq,
                                 const int32_t* row2ts, const int32_t* offsets,
                                 const int32_t* active, const int32_t* meta, int32_t* acc1,
                                 cudaStream_t s);
cudaError_t launch_swiglu_requant(const moe_w8a8_weights* w, const int32_t* acc1,
                                  const int32_t* row2ts, const int32_t* topk_idx,
                                  const float* sx, const int32_t* meta, int max_rows, int8_t* hq,
                                  float* sh, cudaStream_t s);
cudaError_t launch_stream_down(const moe_w8a8_weights* w, int T, const int8_t* hq,
                               const float* sh, const int32_t* row2ts, const float* topk_w,
                               const int32_t* offsets, const int32_t* active, const int32_t* meta,
                               void* o, int32_t* acc2_dbg, cudaStream_t s);
// tensor-core path (kernels_tc.cu)
bool tc_make_weight_maps(moe_w8a8_weights* w);
// dst = src [rows][K] (rows % 256 == 0, K % 128 == 0) in the tiled layout of w_gu_t.
cudaError_t launch_tile_weights(const int8_t* src, int64_t rows, int K, int8_t* dst, cudaStream_t s);
// Certified tensor-core router: approximate logits l~ [T][E] from bf16 X (this
// file's kernels_tc.cu), then per token the candidate experts within the error
// bound, their logits in the stated fp32 order, top-k and gate weights
// (kernels_route.cu).  sel: [T][E] scratch.
bool router_tc_make_maps(moe_w8a8_weights* w);
cudaError_t launch_router_tc(const moe_w8a8_weights* w, const void* x, int T, float* approx, cudaStream_t s);
cudaError_t launch_router_select(const moe_w8a8_weights* w, const void* x, int T, const float* approx,
                                 const float* bias, float* sel, int32_t* idx, float* wts, float* logits_out,
                                 cudaStream_t s);
constexpr int kRouterTcMinTokens = 1024;   // the certified router runs from this many tokens up
bool tc_supported(const moe_w8a8_config& c);
// n_mma back-to-back M=128 N=256 K=32 8-bit MMAs per CTA on `grid` CTAs
// (operands resident in shared memory): the tensor pipe's own rate.
cudaError_t launch_tc_peak(int fmt, int64_t n_mma, int grid, cudaStream_t s);
// pairs != null: run on SM pairs (cta_group::2 MMA, 256-row pair tiles).
cudaError_t launch_tc_gemm1(const moe_w8a8_weights* w, int T, const int8_t* aq, const int32_t* meta,
                            const int32_t* tiles, const int32_t* pairs, const int32_t* offsets,
                            const int32_t* row2ts, const float* sx, float* h32, float* pamax, int32_t* acc_dbg,
                            cudaStream_t s);
cudaError_t launch_requant(const float* h32, const float* pamax, int f, const int32_t* meta,
                           int max_rows, int8_t* hq, float* sh, int fmt, cudaStream_t s);
cudaError_t launch_tc_gemm2(const moe_w8a8_weights* w, int T, const int8_t* hq, const float* sh,
                            const int32_t* meta, const int32_t* tiles, const int32_t* pairs,
                            const int32_t* offsets, const int32_t* row2ts, const float* topk_w, void* o,
                            int32_t* acc_dbg, cudaStream_t s);

// GEMM1 + requantisation of h + GEMM2 in one persistent launch (few rows per
// expert).  sync_words: fused_sync_words(max m-tiles) words, zeroed before the launch.
cudaError_t launch_tc_ffn_fused(const moe_w8a8_weights* w, int T, const int8_t* aq, const int32_t* meta,
                                const int32_t* tiles, const int32_t* offsets, const int32_t* row2ts,
                                const float* sx, const float* topk_w, float* h32, float* pamax, int8_t* hq,
                                float* sh, void* o, int32_t* acc1_dbg, int32_t* acc2_dbg, int32_t* sync_words,
                                cudaStream_t s);
inline size_t fused_sync_words(size_t max_mtiles) { return 2 * max_mtiles + 2; }
constexpr int kFusedMaxRows = 512;   // default: T*k at or below which the tensor path runs the fused launch
// At most this many tokens: the fused launch runs its swapped-operand plan (weights as the MMA's
// 128-row operand, the m-tile's at most 32 token rows as its N = 32 operand), whose partial row
// maxima cover 32 channels each ([rows][f / 32]; otherwise 64: [rows][f / 64]).
constexpr int kFusedSwapTokens = 32;
inline bool fused_swapped(int T) { return T <= kFusedSwapTokens; }

// The per-slot rows o (sorted, [rows][d]) are fp32, or bf16 when o_bf16; the
// expert FFN writes them in the layer's output precision.
cudaError_t launch_combine(const void* o, int o_bf16, const int32_t* ts2row, int T, int k, int d,
                           int out_dtype, void* y, cudaStream_t s);
// The combine over fp32 output rows returned in the fixed blocks of an
// expert-parallel exchange (`offsets` the dispatch's E + 1 row offsets).
cudaError_t launch_combine_blocked(const float* o_blocks, const int32_t* ts2row, const int32_t* offsets,
                                   const EpRanks& ranks, int world, int block_rows, int T, int k, int d,
                                   int out_dtype, void* y, cudaStream_t s);
// Bytes of one per-slot output value: the layer's output precision.
inline size_t o_bytes(const moe_w8a8_config& c) { return c.out_dtype == MOE_BF16 ? 2 : 4; }

}  // namespace moe
