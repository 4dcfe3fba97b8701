// C ABI of the W8A8 MoE layer: argument checks, the prepared-weights handle,
// the workspace layout and the launch sequence of one forward.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <climits>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

moe_status check_config(const moe_w8a8_config* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (!(c->alpha >= 0.0f && c->alpha <= 1.0f)) return MOE_ERR_INVALID_ARG;
    if (c->in_dtype != MOE_F32 && c->in_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->out_dtype != MOE_F32 && c->out_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->renormalize != 0 && c->renormalize != 1) return MOE_ERR_INVALID_ARG;
    if (c->expert_format != MOE_FMT_INT8 && c->expert_format != MOE_FMT_E4M3) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(c->capacity_factor)) return MOE_ERR_INVALID_ARG;
    if (c->d <= 0 || c->f <= 0 || c->n_experts <= 0 || c->top_k <= 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->d % 128 || c->f % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->d > 16384 || c->f > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->n_experts > kMaxE || c->top_k > kMaxK || c->top_k > c->n_experts) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

// Capacity per expert: ceil(cf * T * k / E) in fp64, -1 for none.  Clamped to
// T * k before the conversion (no expert can receive more rows than that, so
// the clamp changes nothing but keeps the conversion defined for large cf).
int capacity_of(const moe_w8a8_config& c, int T) {
    if (!(c.capacity_factor > 0.0f)) return -1;
    const double tk = (double)((int64_t)T * c.top_k);
    const double cap = std::ceil((double)c.capacity_factor * tk / (double)c.n_experts);
    return (int)std::min(cap, tk);
}

// A device pointer the kernels read or write with 16-byte vector accesses.
bool misaligned16(const void* p) { return ((uintptr_t)p & 15) != 0; }

bool tensor_ok(const moe_w8a8_weights* w) { return w->tmaps_ok && tc_supported(w->cfg); }

int choose_path(const moe_w8a8_weights* w, int T) {
    if (w->path != MOE_PATH_AUTO) return w->path;
    if (w->cfg.expert_format == MOE_FMT_E4M3) return MOE_PATH_TENSOR;   // no streaming FP8 path
    if (!tensor_ok(w)) return MOE_PATH_STREAM;
    return (int64_t)T * w->cfg.top_k <= w->stream_max_rows ? MOE_PATH_STREAM : MOE_PATH_TENSOR;
}

// The chosen path can run this handle: the tensor path needs its tensor maps
// and shape, the streaming path INT8 experts.
bool path_ok(const moe_w8a8_weights* w, int T) {
    const int path = choose_path(w, T);
    if (path == MOE_PATH_TENSOR) return tensor_ok(w);
    return w->cfg.expert_format == MOE_FMT_INT8;
}

// The tensor path runs GEMM1, the requantisation of h and GEMM2 as one
// launch up to the handle's row threshold (the routing front end, the
// one-block kernel or the scatter kernel, clears the launch's counters).
// The certified tensor-core router serves large batches with computed logits
// (the one-block routing front end keeps the FMA router).
bool router_tc_ok(const moe_w8a8_weights* w, int T) {
    return w->rt_epad > 0 && T >= kRouterTcMinTokens && !route_small_ok(T, w->cfg.top_k);
}

bool fused_ok(const moe_w8a8_weights* w, int T) {
    return (int64_t)T * w->cfg.top_k <= w->fused_max_rows;
}

void prof_free(moe_w8a8_weights* w) {
    if (!w->prof_events) return;
    for (int i = 0; i < w->prof_max * MOE_N_STAGES * 2; ++i) cudaEventDestroy(w->prof_events[i]);
    delete[] w->prof_events;
    w->prof_events = nullptr;
    w->prof_max = w->prof_n = 0;
}

void free_handle(moe_w8a8_weights* w) {
    if (!w) return;
    prof_free(w);
    cudaFree(w->w_gu);
    cudaFree(w->w_dn);
    cudaFree(w->w_gu_t);
    cudaFree(w->w_dn_t);
    cudaFree(w->sw_gate);
    cudaFree(w->sw_up);
    cudaFree(w->sw_dn);
    cudaFree(w->inv_s);
    cudaFree(w->w_router);
    cudaFree(w->rt_hi);
    cudaFree(w->rt_lo);
    cudaFree(w->rt_wt);
    cudaFree(w->rt_wmax);
    cudaFree(w->status);
    std::free(w->s_host);
    delete w;
}

#define CUDA_TRY(expr)                                  \
    do {                                                \
        cudaError_t err_ = (expr);                      \
        if (err_ != cudaSuccess) return MOE_ERR_CUDA;   \
    } while (0)

}  // namespace

namespace moe {

WsLayout ws_layout(const moe_w8a8_weights* w, int T, WsPart part) {
    const moe_w8a8_config& c = w->cfg;
    const int E = c.n_experts, k = c.top_k, d = c.d, f = c.f;
    const size_t tk = (size_t)T * k;
    const size_t in_b = c.in_dtype == MOE_BF16 ? 2 : 4, out_b = c.out_dtype == MOE_BF16 ? 2 : 4;
    const size_t nblk = (tk + kPermChunk - 1) / kPermChunk;
    const size_t max_tiles = (tk + kTileM - 1) / kTileM + E;
    const bool stream = choose_path(w, T) == MOE_PATH_STREAM;
    const bool fwd = part == WS_FORWARD, route = part == WS_ROUTE, experts = part == WS_EXPERTS;
    WsLayout L{};
    size_t p = 0;
    auto take = [&](size_t bytes) { size_t at = p; p = align_up(p + bytes); return at; };
    L.x_stage = take(fwd ? (size_t)T * d * in_b : 0);
    L.y_stage = take(fwd ? (size_t)T * d * out_b : 0);
    L.logits_stage = take(fwd ? (size_t)T * E * 4 : 0);
    L.bias_stage = take(fwd ? (size_t)E * 4 : 0);
    L.logits = take(experts ? 0 : (size_t)T * E * 4);
    L.logits_sel = take(!experts && router_tc_ok(w, T) ? (size_t)T * E * 4 : 0);
    L.topk_idx = take(tk * 4);
    L.topk_w = take(tk * 4);
    L.hist = take(nblk * E * 4);
    L.offsets = take((size_t)(E + 1) * 4);
    L.meta = take(META_WORDS * 4);
    L.active = take((size_t)E * 4);
    L.tiles = take(max_tiles * 8);
    L.pairs = take(((tk + kPairM - 1) / kPairM + E) * 8);
    L.row2ts = take(tk * 4);
    L.ts2row = take(tk * 4);
    L.xq = take(experts && !stream ? 0 : (size_t)T * d);
    L.sx = take((size_t)T * 4);
    const bool ex = !route;   // expert buffers
    L.aq = take(ex && !stream ? tk * d : 0);
    L.acc1 = take(ex && stream ? tk * 2 * f * 4 : 0);
    L.hq = take(ex ? tk * f : 0);
    L.sh = take(ex ? tk * 4 : 0);
    L.o = take(ex ? tk * d * o_bytes(c) : 0);
    L.h32 = take(ex && !stream ? tk * f * 4 : 0);
    const bool fused = ex && !stream && fused_ok(w, T);
    L.pamax = take(ex && !stream ? tk * (f / (fused && fused_swapped(T) ? 32 : 64)) * 4 : 0);
    L.fused_sync = take(fused ? fused_sync_words(max_tiles) * 4 : 0);
    L.fused_words = fused ? (int)fused_sync_words(max_tiles) : 0;
    L.total = p;
    return L;
}

}  // namespace moe

namespace moe {
namespace {

// fp32 -> bf16 bits, round to nearest even (finite values).
uint16_t bf16_rn(float v) {
    uint32_t b;
    std::memcpy(&b, &v, 4);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

float bf16_value(uint16_t h) {
    const uint32_t b = (uint32_t)h << 16;
    float v;
    std::memcpy(&v, &b, 4);
    return v;
}

// Tables of the certified tensor-core router (bf16 X, renormalised gate):
// W_g [d][E] -> hi, lo [epad][d] bf16 with hi = bf16(w), lo = bf16(w - hi)
// (w - hi is exact in fp32), W_g transposed [E][d], max_e |W_g[j][e]| [d].
// Leaves rt_epad = 0 (FMA router only) when the layer does not qualify or a
// step fails.
void prepare_router_tc(moe_w8a8_weights* w, cudaStream_t s) {
    const moe_w8a8_config& c = w->cfg;
    const int d = c.d, E = c.n_experts;
    w->rt_epad = 0;
    if (c.in_dtype != MOE_BF16 || c.renormalize != 1 || d % 128 != 0 || E > 256) return;
    const int epad = E <= 64 ? 64 : (E <= 128 ? 128 : 256);
    std::vector<float> wg((size_t)d * E), wt((size_t)E * d), wmax(d, 0.0f);
    std::vector<uint16_t> hi((size_t)epad * d, 0), lo((size_t)epad * d, 0);
    if (cudaMemcpyAsync(wg.data(), w->w_router, wg.size() * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return;
    // wt and wmax lane-interleaved: channel j = 32 i + p at [i / 4][p][i % 4]
    auto lane_pos = [](int j) { const int i = j / 32, p = j % 32; return (size_t)(i / 4) * 128 + p * 4 + i % 4; };
    std::vector<float> wmax_lin(d, 0.0f);
    for (int j = 0; j < d; ++j)
        for (int e = 0; e < E; ++e) {
            const float v = wg[(size_t)j * E + e];
            const uint16_t h = bf16_rn(v);
            hi[(size_t)e * d + j] = h;
            lo[(size_t)e * d + j] = bf16_rn(v - bf16_value(h));
            wt[(size_t)e * d + lane_pos(j)] = v;
            wmax_lin[j] = std::max(wmax_lin[j], std::fabs(v));
        }
    for (int j = 0; j < d; ++j) wmax[lane_pos(j)] = wmax_lin[j];
    bool ok = cudaMalloc(&w->rt_hi, hi.size() * 2) == cudaSuccess &&
              cudaMalloc(&w->rt_lo, lo.size() * 2) == cudaSuccess &&
              cudaMalloc(&w->rt_wt, wt.size() * 4) == cudaSuccess &&
              cudaMalloc(&w->rt_wmax, wmax.size() * 4) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(w->rt_hi, hi.data(), hi.size() * 2, cudaMemcpyHostToDevice, s) == cudaSuccess &&
         cudaMemcpyAsync(w->rt_lo, lo.data(), lo.size() * 2, cudaMemcpyHostToDevice, s) == cudaSuccess &&
         cudaMemcpyAsync(w->rt_wt, wt.data(), wt.size() * 4, cudaMemcpyHostToDevice, s) == cudaSuccess &&
         cudaMemcpyAsync(w->rt_wmax, wmax.data(), wmax.size() * 4, cudaMemcpyHostToDevice, s) == cudaSuccess &&
         cudaStreamSynchronize(s) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return;
    }
    w->rt_epad = epad;
    if (!router_tc_make_maps(w)) w->rt_epad = 0;
}

}  // namespace
}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_OOM: return "device allocation failed";
    }
    return "unknown status";
}

moe_status moe_w8a8_calibrate_absmax(const void* x, int64_t rows, int32_t d, int32_t dtype,
                                     float* absmax, moe_stream_t stream) {
    if (!absmax || rows < 0 || (rows > 0 && !x)) return MOE_ERR_INVALID_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (d <= 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (launch_calib_absmax(x, rows, d, dtype, absmax, (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"

namespace {

// Prepare experts [e_first, e_first + n_local) of the layer (all of them for
// the single-GPU handle).  gateup_absmax: the layer's aw (max over ALL experts)
// on the device, or null to take it from the given experts.
moe_status prepare_impl(const moe_w8a8_config* cfg, int e_first, int n_local, const float* w_gate,
                        const float* w_up, const float* w_down, const float* w_router, const float* act_absmax,
                        const float* gateup_absmax, moe_stream_t stream, moe_w8a8_weights** out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!w_gate || !w_up || !w_down || !w_router || !act_absmax) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_config c = *cfg;
    if (e_first < 0 || n_local <= 0 || e_first + n_local > c.n_experts) return MOE_ERR_INVALID_ARG;
    const int E = n_local, d = c.d, f = c.f;   // expert arrays hold the n_local experts
    const int E_layer = c.n_experts;           // the router scores all of the layer's experts
    cudaStream_t s = (cudaStream_t)stream;

    moe_w8a8_weights* w = new moe_w8a8_weights();
    w->cfg = c;
    w->ep_first = e_first;
    w->n_local = n_local;
    w->path = MOE_PATH_AUTO;
    w->stream_max_rows = 32;   // measured crossover: streaming wins up to T*k = 32 rows
    w->wait_budget_ns = 2000000000ull;
    w->test_skip_ready = -1;
    w->fused_max_rows = kFusedMaxRows;
    w->cta_pairs = 2;
    if (cudaGetDevice(&w->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&w->num_sms, cudaDevAttrMultiProcessorCount, w->device) != cudaSuccess) {
        free_handle(w);
        return MOE_ERR_CUDA;
    }
    const size_t n_gu = (size_t)E * 2 * f * d, n_dn = (size_t)E * d * f;
    bool ok = cudaMalloc(&w->w_gu, n_gu) == cudaSuccess && cudaMalloc(&w->w_dn, n_dn) == cudaSuccess &&
              cudaMalloc(&w->sw_gate, (size_t)E * f * 4) == cudaSuccess &&
              cudaMalloc(&w->sw_up, (size_t)E * f * 4) == cudaSuccess &&
              cudaMalloc(&w->sw_dn, (size_t)E * d * 4) == cudaSuccess &&
              cudaMalloc(&w->inv_s, (size_t)d * 4) == cudaSuccess &&
              cudaMalloc(&w->w_router, (size_t)d * E_layer * 4) == cudaSuccess &&
              cudaMalloc(&w->status, 64) == cudaSuccess;
    w->s_host = (float*)std::malloc((size_t)d * 4);
    float* tmp = nullptr;   // aw [d] then s [d] on the device
    ok = ok && w->s_host && cudaMalloc(&tmp, (size_t)2 * d * 4) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        cudaFree(tmp);
        free_handle(w);
        return MOE_ERR_OOM;
    }
    auto fail = [&](moe_status code) {
        cudaFree(tmp);
        free_handle(w);
        return code;
    };
    float* aw_dev = tmp;
    float* s_dev = tmp + d;
    if (cudaMemsetAsync(w->status, 0, 64, s) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (!gateup_absmax && (cudaMemsetAsync(aw_dev, 0, (size_t)d * 4, s) != cudaSuccess ||
                           launch_gateup_input_absmax(w_gate, w_up, E, d, f, aw_dev, s) != cudaSuccess))
        return fail(MOE_ERR_CUDA);
    std::vector<float> aw(d), ax(d), inv(d);
    if (cudaMemcpyAsync(aw.data(), gateup_absmax ? gateup_absmax : aw_dev, (size_t)d * 4, cudaMemcpyDeviceToHost,
                        s) != cudaSuccess ||
        cudaMemcpyAsync(ax.data(), act_absmax, (size_t)d * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    // SmoothQuant scales, fp64 on the host: s_j = ax^alpha / aw^(1-alpha), both
    // statistics floored at 1e-5; inv_s_j = fp32(1 / s_j).
    const double a = (double)c.alpha;
    const double floor_v = (double)1e-5f;
    for (int j = 0; j < d; ++j) {
        const double xv = ax[j] > 1e-5f ? (double)ax[j] : floor_v;
        const double wv = aw[j] > 1e-5f ? (double)aw[j] : floor_v;
        w->s_host[j] = (float)(std::pow(xv, a) / std::pow(wv, 1.0 - a));
        inv[j] = (float)(1.0 / (double)w->s_host[j]);
    }
    if (cudaMemcpyAsync(s_dev, w->s_host, (size_t)d * 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(w->inv_s, inv.data(), (size_t)d * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    // gate -> rows [blk*256, blk*256+128), up -> rows [blk*256+128, blk*256+256)
    const int fmt = c.expert_format;
    if (launch_quantize_channels(w_gate, s_dev, E, d, f, w->w_gu, 2 * f, kGuBlock, 2 * kGuBlock, 0,
                                 w->sw_gate, fmt, s) != cudaSuccess ||
        launch_quantize_channels(w_up, s_dev, E, d, f, w->w_gu, 2 * f, kGuBlock, 2 * kGuBlock,
                                 kGuBlock, w->sw_up, fmt, s) != cudaSuccess ||
        launch_quantize_channels(w_down, nullptr, E, f, d, w->w_dn, d, d, d, 0, w->sw_dn, fmt, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(w->w_router, w_router, (size_t)d * E_layer * 4, cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    // the tensor-core kernels' tiled copies (only for layers they serve)
    if (tc_supported(c)) {
        if (cudaMalloc(&w->w_gu_t, n_gu) != cudaSuccess || cudaMalloc(&w->w_dn_t, n_dn) != cudaSuccess) {
            cudaGetLastError();
            return fail(MOE_ERR_OOM);
        }
        if (launch_tile_weights(w->w_gu, (int64_t)E * 2 * f, d, w->w_gu_t, s) != cudaSuccess ||
            launch_tile_weights(w->w_dn, (int64_t)E * d, f, w->w_dn_t, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        w->tmaps_ok = tc_make_weight_maps(w);
    }
    prepare_router_tc(w, s);
    cudaFree(tmp);
    *out = w;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_w8a8_prepare(const moe_w8a8_config* cfg, const float* w_gate, const float* w_up,
                            const float* w_down, const float* w_router, const float* act_absmax,
                            moe_stream_t stream, moe_w8a8_weights** out) {
    if (!cfg) {
        if (out) *out = nullptr;
        return MOE_ERR_INVALID_ARG;
    }
    return prepare_impl(cfg, 0, cfg->n_experts, w_gate, w_up, w_down, w_router, act_absmax, nullptr, stream, out);
}

size_t moe_w8a8_workspace_size(const moe_w8a8_weights* w, int32_t max_tokens) {
    if (!w || max_tokens < 0) return 0;
    return ws_layout(w, max_tokens).total;
}

}  // extern "C"

namespace {

// One call's launch context: the handle whose cfg describes the call (for the
// expert side of the expert-parallel layer a view of it), the workspace and its
// layout, the debug buffers and the per-stage profiling marks.
struct Run {
    const moe_w8a8_weights* w;
    WsLayout L;
    char* ws;
    const moe_w8a8_debug* dbg;
    cudaStream_t s;
    bool prof;
    int launches = 0;

    Run(const moe_w8a8_weights* w_, const WsLayout& L_, char* ws_, const moe_w8a8_debug* dbg_, cudaStream_t s_)
        : w(w_), L(L_), ws(ws_), dbg(dbg_), s(s_), prof(w_->prof_events && w_->prof_n < w_->prof_max) {}
    template <class V>
    V* at(size_t off) const { return reinterpret_cast<V*>(ws + off); }
    void mark(int stage, int edge) const {
        if (prof && (w->prof_mask >> stage & 1u))
            cudaEventRecord(w->prof_events[(w->prof_n * MOE_N_STAGES + stage) * 2 + edge], s);
    }
    void empty_stage(int stage) const { mark(stage, 0); mark(stage, 1); }
};

// Router, top-k and the expert-major permutation (with capacity) of T tokens
// over the layer's E experts.
moe_status route_stage(Run& r, const void* x, int T, const float* bias, const float* given_logits, int path) {
    const moe_w8a8_weights* w = r.w;
    const moe_w8a8_config& c = w->cfg;
    const int E = c.n_experts, k = c.top_k, d = c.d;
    const WsLayout& L = r.L;
    cudaStream_t s = r.s;
    float* logits = r.at<float>(L.logits);
    int32_t* idx = r.at<int32_t>(L.topk_idx);
    float* wts = r.at<float>(L.topk_w);
    int32_t* offsets = r.at<int32_t>(L.offsets);
    int32_t* meta = r.at<int32_t>(L.meta);
    int32_t* active = r.at<int32_t>(L.active);
    int32_t* tiles = r.at<int32_t>(L.tiles);
    int32_t* row2ts = r.at<int32_t>(L.row2ts);
    int32_t* ts2row = r.at<int32_t>(L.ts2row);
    float* dbg_logits = r.dbg ? r.dbg->logits : nullptr;

    const float* lsrc = given_logits;
    const bool certified = !lsrc && router_tc_ok(w, T);
    if (certified) {
        // approximate logits on the tensor cores, then per token the candidates'
        // logits in the stated order, top-k and gate weights
        r.mark(MOE_STAGE_ROUTER, 0);
        CUDA_TRY(launch_router_tc(w, x, T, logits, s));
        r.mark(MOE_STAGE_ROUTER, 1);
        r.mark(MOE_STAGE_TOPK, 0);
        CUDA_TRY(launch_router_select(w, x, T, logits, bias, r.at<float>(L.logits_sel), idx, wts, dbg_logits, s));
        r.mark(MOE_STAGE_TOPK, 1);
        r.launches += 2;
    } else if (!lsrc) {
        r.mark(MOE_STAGE_ROUTER, 0);
        CUDA_TRY(launch_router_logits(x, c.in_dtype, w->w_router, T, d, E, logits, s));
        r.mark(MOE_STAGE_ROUTER, 1);
        ++r.launches;
        lsrc = logits;
    } else {
        r.empty_stage(MOE_STAGE_ROUTER);
    }
    const bool fused = path == MOE_PATH_TENSOR && L.fused_words > 0;
    int32_t* zero_words = fused ? r.at<int32_t>(L.fused_sync) : nullptr;
    const int n_zero = fused ? L.fused_words : 0;
    if (certified) {
        r.mark(MOE_STAGE_PERMUTE, 0);
        CUDA_TRY(launch_permute(idx, T, k, E, capacity_of(c, T), r.at<int32_t>(L.hist), offsets, row2ts, ts2row,
                                meta, active, tiles, r.at<int32_t>(L.pairs), s, zero_words, n_zero));
        r.mark(MOE_STAGE_PERMUTE, 1);
        r.launches += 2;
    } else if (route_small_ok(T, k)) {
        // top-k, histogram, scan and scatter in one block
        r.mark(MOE_STAGE_TOPK, 0);
        CUDA_TRY(launch_route_small(lsrc, bias, T, E, k, c.renormalize, capacity_of(c, T), idx, wts, dbg_logits,
                                    offsets, row2ts, ts2row, meta, active, tiles, r.at<int32_t>(L.pairs), zero_words,
                                    n_zero, s));
        r.mark(MOE_STAGE_TOPK, 1);
        r.empty_stage(MOE_STAGE_PERMUTE);
        ++r.launches;
    } else {
        r.mark(MOE_STAGE_TOPK, 0);
        CUDA_TRY(launch_topk(lsrc, bias, T, E, k, c.renormalize, idx, wts, dbg_logits, s));
        r.mark(MOE_STAGE_TOPK, 1);
        ++r.launches;
        r.mark(MOE_STAGE_PERMUTE, 0);
        CUDA_TRY(launch_permute(idx, T, k, E, capacity_of(c, T), r.at<int32_t>(L.hist), offsets, row2ts, ts2row,
                                meta, active, tiles, r.at<int32_t>(L.pairs), s, zero_words, n_zero));
        r.mark(MOE_STAGE_PERMUTE, 1);
        r.launches += 2;
    }
    return MOE_OK;
}

// Smoothing and per-token quantisation; the codes of each kept (t, slot) go
// to its sorted row of aq (row stride aq_ld), followed by the expert-parallel
// trailer when `trailer` is set.
moe_status quant_stage(Run& r, const void* x, int T, int8_t* aq, int64_t aq_ld, bool trailer, int fmt) {
    const moe_w8a8_weights* w = r.w;
    const moe_w8a8_config& c = w->cfg;
    const WsLayout& L = r.L;
    // the per-token codes are read by the streaming path and the debug copy;
    // the tensor path and the expert-parallel send rows use the sorted copies
    const bool need_xq = !aq || (r.dbg && r.dbg->xq);
    r.mark(MOE_STAGE_QUANT, 0);
    CUDA_TRY(launch_smooth_quant(x, c.in_dtype, w->inv_s, w->act_clip, T, c.d, c.top_k, r.at<int32_t>(L.ts2row),
                                 need_xq ? r.at<int8_t>(L.xq) : nullptr, r.at<float>(L.sx), aq, aq_ld,
                                 trailer ? r.at<float>(L.topk_w) : nullptr,
                                 trailer ? r.at<int32_t>(L.topk_idx) : nullptr, fmt, r.s));
    r.mark(MOE_STAGE_QUANT, 1);
    ++r.launches;
    return MOE_OK;
}

// The experts of T*k sorted rows (codes in xq by token for the streaming path,
// in aq by row for the tensor path; sx, topk_w, topk_idx by token / (t, slot))
// to the per-row outputs O.
moe_status expert_stage(Run& r, int T, int path) {
    const moe_w8a8_weights* w = r.w;
    const moe_w8a8_config& c = w->cfg;
    const int k = c.top_k, f = c.f;
    const WsLayout& L = r.L;
    cudaStream_t s = r.s;
    const moe_w8a8_debug* dbg = r.dbg;
    const size_t tk = (size_t)T * k;
    int32_t* idx = r.at<int32_t>(L.topk_idx);
    float* wts = r.at<float>(L.topk_w);
    int32_t* offsets = r.at<int32_t>(L.offsets);
    int32_t* meta = r.at<int32_t>(L.meta);
    int32_t* active = r.at<int32_t>(L.active);
    int32_t* tiles = r.at<int32_t>(L.tiles);
    int32_t* row2ts = r.at<int32_t>(L.row2ts);
    float* sx = r.at<float>(L.sx);
    int8_t* hq = r.at<int8_t>(L.hq);
    float* sh = r.at<float>(L.sh);
    void* o = r.at<void>(L.o);
    if (path == MOE_PATH_STREAM) {
        int32_t* acc1 = r.at<int32_t>(L.acc1);
        r.mark(MOE_STAGE_GEMM1, 0);
        CUDA_TRY(launch_stream_gateup(w, T, r.at<int8_t>(L.xq), row2ts, offsets, active, meta, acc1, s));
        r.mark(MOE_STAGE_GEMM1, 1);
        r.mark(MOE_STAGE_REQUANT, 0);
        CUDA_TRY(launch_swiglu_requant(w, acc1, row2ts, idx, sx, meta, (int)tk, hq, sh, s));
        r.mark(MOE_STAGE_REQUANT, 1);
        r.mark(MOE_STAGE_GEMM2, 0);
        CUDA_TRY(launch_stream_down(w, T, hq, sh, row2ts, wts, offsets, active, meta, o,
                                    dbg ? dbg->acc2 : nullptr, s));
        r.mark(MOE_STAGE_GEMM2, 1);
        r.launches += 3;
        if (dbg && dbg->acc1)
            CUDA_TRY(cudaMemcpyAsync(dbg->acc1, acc1, tk * 2 * f * 4, cudaMemcpyDeviceToDevice, s));
        return MOE_OK;
    }
    int8_t* aq = r.at<int8_t>(L.aq);
    if (L.fused_words > 0) {
        // few rows per expert: GEMM1, requantisation and GEMM2 in one launch
        // (its time is reported as the GEMM1 stage)
        r.mark(MOE_STAGE_GEMM1, 0);
        CUDA_TRY(launch_tc_ffn_fused(w, T, aq, meta, tiles, offsets, row2ts, sx, wts, r.at<float>(L.h32),
                                     r.at<float>(L.pamax), hq, sh, o, dbg ? dbg->acc1 : nullptr,
                                     dbg ? dbg->acc2 : nullptr, r.at<int32_t>(L.fused_sync), s));
        r.mark(MOE_STAGE_GEMM1, 1);
        r.empty_stage(MOE_STAGE_REQUANT);
        r.empty_stage(MOE_STAGE_GEMM2);
        r.launches += 1;
        return MOE_OK;
    }
    r.mark(MOE_STAGE_GEMM1, 0);
    // SM pairs (256-row tiles) when asked to, or by default when the rows per
    // expert fill such tiles on average (a pair tile's second half is wasted
    // MMA work on an expert's last rows)
    const bool pair = w->cta_pairs == 1 || (w->cta_pairs == 2 && tk >= (size_t)kPairM * w->cfg.n_experts);
    const int32_t* pairs = pair ? r.at<int32_t>(L.pairs) : nullptr;
    CUDA_TRY(launch_tc_gemm1(w, T, aq, meta, tiles, pairs, offsets, row2ts, sx, r.at<float>(L.h32), r.at<float>(L.pamax),
                             dbg ? dbg->acc1 : nullptr, s));
    r.mark(MOE_STAGE_GEMM1, 1);
    r.mark(MOE_STAGE_REQUANT, 0);
    CUDA_TRY(launch_requant(r.at<float>(L.h32), r.at<float>(L.pamax), f, meta, (int)tk, hq, sh, c.expert_format, s));
    r.mark(MOE_STAGE_REQUANT, 1);
    r.mark(MOE_STAGE_GEMM2, 0);
    CUDA_TRY(launch_tc_gemm2(w, T, hq, sh, meta, tiles, pairs, offsets, row2ts, wts, o, dbg ? dbg->acc2 : nullptr,
                             s));
    r.mark(MOE_STAGE_GEMM2, 1);
    r.launches += 3;
    return MOE_OK;
}

// Copies of the intermediates a debug struct asks for (T tokens, k slots,
// E experts in the offsets array; token codes and expert buffers if present).
moe_status debug_stage(Run& r, int T, int k, int E, bool token_codes, bool expert_bufs) {
    const moe_w8a8_debug* dbg = r.dbg;
    if (!dbg) return MOE_OK;
    const WsLayout& L = r.L;
    const size_t tk = (size_t)T * k;
    const int d = r.w->cfg.d, f = r.w->cfg.f;
    auto cp = [&](void* dst, size_t off, size_t bytes) {
        return dst ? cudaMemcpyAsync(dst, r.ws + off, bytes, cudaMemcpyDeviceToDevice, r.s) : cudaSuccess;
    };
    CUDA_TRY(cp(dbg->topk_idx, L.topk_idx, tk * 4));
    CUDA_TRY(cp(dbg->topk_w, L.topk_w, tk * 4));
    CUDA_TRY(cp(dbg->offsets, L.offsets, (size_t)(E + 1) * 4));
    CUDA_TRY(cp(dbg->row2ts, L.row2ts, tk * 4));
    CUDA_TRY(cp(dbg->ts2row, L.ts2row, tk * 4));
    if (token_codes) CUDA_TRY(cp(dbg->xq, L.xq, (size_t)T * d));
    CUDA_TRY(cp(dbg->sx, L.sx, (size_t)T * 4));
    if (expert_bufs) {
        CUDA_TRY(cp(dbg->hq, L.hq, tk * f));
        CUDA_TRY(cp(dbg->sh, L.sh, tk * 4));
        CUDA_TRY(cp(dbg->o, L.o, tk * d * o_bytes(r.w->cfg)));
    }
    return MOE_OK;
}

#define MOE_TRY(expr)                          \
    do {                                       \
        moe_status st_ = (expr);               \
        if (st_ != MOE_OK) return st_;         \
    } while (0)

moe_status forward_impl(const moe_w8a8_weights* w, const void* x, int T, const float* bias,
                        const float* given_logits, void* y, char* ws, const moe_w8a8_debug* dbg, cudaStream_t s) {
    const moe_w8a8_config& c = w->cfg;
    const int path = choose_path(w, T);
    Run r(w, ws_layout(w, T), ws, dbg, s);
    MOE_TRY(route_stage(r, x, T, bias, given_logits, path));
    if (path == MOE_PATH_STREAM)
        MOE_TRY(quant_stage(r, x, T, nullptr, c.d, false, MOE_FMT_INT8));
    else
        MOE_TRY(quant_stage(r, x, T, r.at<int8_t>(r.L.aq), c.d, false, c.expert_format));
    MOE_TRY(expert_stage(r, T, path));
    r.mark(MOE_STAGE_COMBINE, 0);
    CUDA_TRY(launch_combine(r.at<void>(r.L.o), c.out_dtype == MOE_BF16, r.at<int32_t>(r.L.ts2row), T, c.top_k, c.d,
                            c.out_dtype, y, s));
    r.mark(MOE_STAGE_COMBINE, 1);
    ++r.launches;
    moe_w8a8_weights* mw = const_cast<moe_w8a8_weights*>(w);
    if (r.prof) ++mw->prof_n;
    MOE_TRY(debug_stage(r, T, c.top_k, c.n_experts, true, true));
    mw->last_launches = r.launches;
    return MOE_OK;
}

// The handle holds every expert of the layer (not an expert-parallel shard).
bool holds_all_experts(const moe_w8a8_weights* w) { return w->ep_first == 0 && w->n_local == w->cfg.n_experts; }

// The current device is the one the handle's weights live on.
bool on_handle_device(const moe_w8a8_weights* w) {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess && dev == w->device;
}

// The expert side of the expert-parallel layer: the held experts as a layer of
// n_local experts with one slot per row, no capacity, no router and no
// profiling (the kernels index scales and gate weights by row).
moe_w8a8_weights expert_view(const moe_w8a8_weights* w) {
    moe_w8a8_weights v = *w;
    v.cfg.n_experts = w->n_local;
    v.cfg.top_k = 1;
    v.cfg.capacity_factor = 0.0f;
    v.ep_first = 0;
    v.rt_epad = 0;
    v.prof_events = nullptr;
    v.prof_max = v.prof_n = 0;
    return v;
}

}  // namespace

extern "C" {

moe_status moe_w8a8_forward(const moe_w8a8_weights* w, const void* x, int32_t T,
                            const float* router_bias, const float* router_logits, void* y,
                            void* workspace, size_t workspace_bytes, const moe_w8a8_debug* dbg,
                            moe_stream_t stream) {
    if (!w || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !y || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign || misaligned16(x) || misaligned16(y) || misaligned16(router_bias) ||
        misaligned16(router_logits))
        return MOE_ERR_INVALID_ARG;
    if (!holds_all_experts(w) || !on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    if (!path_ok(w, T)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < ws_layout(w, T).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return forward_impl(w, x, T, router_bias, router_logits, y, (char*)workspace, dbg,
                        (cudaStream_t)stream);
}

moe_status moe_w8a8_forward_host(const moe_w8a8_weights* w, const void* x_host, int32_t T,
                                 const float* router_bias_host, const float* router_logits_host,
                                 void* y_host, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream) {
    if (!w || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x_host || !y_host || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign) return MOE_ERR_INVALID_ARG;
    if (!holds_all_experts(w) || !on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    if (!path_ok(w, T)) return MOE_ERR_UNSUPPORTED_SHAPE;
    const WsLayout L = ws_layout(w, T);
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const moe_w8a8_config& c = w->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    const size_t in_b = c.in_dtype == MOE_BF16 ? 2 : 4, out_b = c.out_dtype == MOE_BF16 ? 2 : 4;
    CUDA_TRY(cudaMemcpyAsync(ws + L.x_stage, x_host, (size_t)T * c.d * in_b, cudaMemcpyHostToDevice, s));
    const float* lg = nullptr;
    const float* bs = nullptr;
    if (router_logits_host) {
        CUDA_TRY(cudaMemcpyAsync(ws + L.logits_stage, router_logits_host, (size_t)T * c.n_experts * 4,
                                 cudaMemcpyHostToDevice, s));
        lg = (const float*)(ws + L.logits_stage);
    }
    if (router_bias_host) {
        CUDA_TRY(cudaMemcpyAsync(ws + L.bias_stage, router_bias_host, (size_t)c.n_experts * 4,
                                 cudaMemcpyHostToDevice, s));
        bs = (const float*)(ws + L.bias_stage);
    }
    moe_status st = forward_impl(w, ws + L.x_stage, T, bs, lg, ws + L.y_stage, ws, nullptr, s);
    if (st != MOE_OK) return st;
    CUDA_TRY(cudaMemcpyAsync(y_host, ws + L.y_stage, (size_t)T * c.d * out_b, cudaMemcpyDeviceToHost, s));
    return MOE_OK;
}

moe_status moe_w8a8_set_path(moe_w8a8_weights* w, int32_t path) {
    if (!w || path < MOE_PATH_AUTO || path > MOE_PATH_TENSOR) return MOE_ERR_INVALID_ARG;
    w->path = path;
    return MOE_OK;
}

moe_status moe_w8a8_set_stream_threshold(moe_w8a8_weights* w, int32_t max_rows) {
    if (!w || max_rows < 0) return MOE_ERR_INVALID_ARG;
    w->stream_max_rows = max_rows;
    return MOE_OK;
}

moe_status moe_w8a8_set_cta_pairs(moe_w8a8_weights* w, int32_t mode) {
    if (!w || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
    w->cta_pairs = mode;
    return MOE_OK;
}

moe_status moe_w8a8_set_fused_threshold(moe_w8a8_weights* w, int64_t max_rows) {
    if (!w || max_rows < 0) return MOE_ERR_INVALID_ARG;
    w->fused_max_rows = max_rows;
    return MOE_OK;
}

moe_status moe_w8a8_set_wait_budget(moe_w8a8_weights* w, int64_t ns) {
    if (!w || ns < 1000000 || ns > 60000000000ll) return MOE_ERR_INVALID_ARG;
    w->wait_budget_ns = (uint64_t)ns;
    return MOE_OK;
}

moe_status moe_w8a8_test_withhold_release(moe_w8a8_weights* w, int32_t m_tile) {
    if (!w || m_tile < -1) return MOE_ERR_INVALID_ARG;
    w->test_skip_ready = m_tile;
    return MOE_OK;
}

moe_status moe_w8a8_set_act_clip(moe_w8a8_weights* w, float clip) {
    if (!w || !(clip >= 0.0f) || !std::isfinite(clip)) return MOE_ERR_INVALID_ARG;
    w->act_clip = clip;
    return MOE_OK;
}

moe_status moe_w8a8_calibrate_act_clip(const moe_w8a8_weights* w, const void* x, int64_t rows,
                                       int32_t dtype, double percent, float* clip_host,
                                       moe_stream_t stream) {
    if (!w || !clip_host || rows <= 0 || !x) return MOE_ERR_INVALID_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (!(percent > 0.0 && percent <= 100.0)) return MOE_ERR_INVALID_ARG;
    const int d = w->cfg.d;
    const int64_t n = rows * d;
    cudaStream_t s = (cudaStream_t)stream;
    float* dev = nullptr;
    if (cudaMalloc(&dev, (size_t)n * 4) != cudaSuccess) return MOE_ERR_OOM;
    std::vector<float> a((size_t)n);
    cudaError_t err = launch_scaled_abs(x, rows, d, dtype, w->inv_s, dev, s);
    if (err == cudaSuccess) err = cudaMemcpyAsync(a.data(), dev, (size_t)n * 4, cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    cudaFree(dev);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    // nearest rank: the ceil(percent/100 * n)-th smallest value
    int64_t rank = (int64_t)std::ceil(percent / 100.0 * (double)n);
    rank = std::min<int64_t>(std::max<int64_t>(rank, 1), n);
    std::nth_element(a.begin(), a.begin() + (rank - 1), a.end());
    *clip_host = a[(size_t)(rank - 1)];
    return MOE_OK;
}

moe_status moe_w8a8_get_smooth_scales(const moe_w8a8_weights* w, float* s_host) {
    if (!w || !s_host) return MOE_ERR_INVALID_ARG;
    std::memcpy(s_host, w->s_host, (size_t)w->cfg.d * 4);
    return MOE_OK;
}

moe_status moe_w8a8_export_weights(const moe_w8a8_weights* w, int8_t* wq_gate, int8_t* wq_up,
                                   float* sw_gate, float* sw_up, int8_t* wq_down, float* sw_down,
                                   float* inv_s, moe_stream_t stream) {
    if (!w) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_config& c = w->cfg;
    const int E = w->n_local, d = c.d, f = c.f;
    cudaStream_t s = (cudaStream_t)stream;
    if (wq_gate || wq_up) CUDA_TRY(launch_export_gateup(w->w_gu, E, d, f, wq_gate, wq_up, s));
    auto cp = [&](void* dst, const void* src, size_t bytes) {
        return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s) : cudaSuccess;
    };
    CUDA_TRY(cp(sw_gate, w->sw_gate, (size_t)E * f * 4));
    CUDA_TRY(cp(sw_up, w->sw_up, (size_t)E * f * 4));
    CUDA_TRY(cp(wq_down, w->w_dn, (size_t)E * d * f));
    CUDA_TRY(cp(sw_down, w->sw_dn, (size_t)E * d * 4));
    CUDA_TRY(cp(inv_s, w->inv_s, (size_t)d * 4));
    return MOE_OK;
}

moe_status moe_w8a8_check_status(const moe_w8a8_weights* w, moe_stream_t stream) {
    if (!w) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    int32_t word = 0;
    if (cudaMemcpy(&word, w->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(w->status, 0, 64) != cudaSuccess) return MOE_ERR_CUDA;
        return word == MOE_ERR_INVALID_ARG ? MOE_ERR_INVALID_ARG : MOE_ERR_TIMEOUT;
    }
    return MOE_OK;
}

moe_status moe_w8a8_status_words(const moe_w8a8_weights* w, int32_t* words_host, int32_t n,
                                 moe_stream_t stream) {
    if (!w || !words_host || n < 0 || n > 16) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (n && cudaMemcpy(words_host, w->status, (size_t)n * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

void moe_w8a8_destroy(moe_w8a8_weights* w) { free_handle(w); }

moe_status moe_w8a8_profile_start(moe_w8a8_weights* w, int32_t max_forwards) {
    return moe_w8a8_profile_start_stages(w, max_forwards, (1u << MOE_N_STAGES) - 1u);
}

moe_status moe_w8a8_profile_start_stages(moe_w8a8_weights* w, int32_t max_forwards, uint32_t stage_mask) {
    if (!w || max_forwards <= 0 || stage_mask == 0 || (stage_mask >> MOE_N_STAGES) != 0) return MOE_ERR_INVALID_ARG;
    prof_free(w);
    const int n = max_forwards * MOE_N_STAGES * 2;
    w->prof_events = new cudaEvent_t[n];
    for (int i = 0; i < n; ++i) {
        if (cudaEventCreate(&w->prof_events[i]) != cudaSuccess) {
            for (int j = 0; j < i; ++j) cudaEventDestroy(w->prof_events[j]);
            delete[] w->prof_events;
            w->prof_events = nullptr;
            return MOE_ERR_CUDA;
        }
    }
    w->prof_max = max_forwards;
    w->prof_n = 0;
    w->prof_mask = stage_mask;
    return MOE_OK;
}

int32_t moe_w8a8_profile_read(moe_w8a8_weights* w, float* ms_host, int32_t capacity) {
    if (!w || !ms_host || capacity < 0 || !w->prof_events) return -1;
    const int n = w->prof_n < capacity ? w->prof_n : capacity;
    for (int i = 0; i < n; ++i)
        for (int st = 0; st < MOE_N_STAGES; ++st) {
            if (!(w->prof_mask >> st & 1u)) {
                ms_host[i * MOE_N_STAGES + st] = 0.0f;
                continue;
            }
            cudaEvent_t a = w->prof_events[(i * MOE_N_STAGES + st) * 2];
            cudaEvent_t b = w->prof_events[(i * MOE_N_STAGES + st) * 2 + 1];
            if (cudaEventSynchronize(b) != cudaSuccess) return -1;
            float ms = 0.0f;
            if (cudaEventElapsedTime(&ms, a, b) != cudaSuccess) return -1;
            ms_host[i * MOE_N_STAGES + st] = ms;
        }
    return n;
}

moe_status moe_w8a8_profile_stop(moe_w8a8_weights* w) {
    if (!w) return MOE_ERR_INVALID_ARG;
    prof_free(w);
    return MOE_OK;
}

// ---------------------------------------------------------------- expert parallelism

int32_t moe_w8a8_ep_row_bytes(const moe_w8a8_weights* w) { return w ? w->cfg.d + kEpTrailerBytes : 0; }

moe_status moe_w8a8_gateup_absmax(const moe_w8a8_config* cfg, int32_t n_local, const float* w_gate,
                                  const float* w_up, float* aw, moe_stream_t stream) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!w_gate || !w_up || !aw || n_local <= 0 || n_local > cfg->n_experts) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    CUDA_TRY(cudaMemsetAsync(aw, 0, (size_t)cfg->d * 4, s));
    CUDA_TRY(launch_gateup_input_absmax(w_gate, w_up, n_local, cfg->d, cfg->f, aw, s));
    return MOE_OK;
}

moe_status moe_w8a8_prepare_shard(const moe_w8a8_config* cfg, int32_t expert_first, int32_t n_local,
                                  const float* w_gate, const float* w_up, const float* w_down,
                                  const float* w_router, const float* act_absmax, const float* gateup_absmax,
                                  moe_stream_t stream, moe_w8a8_weights** out) {
    if (out) *out = nullptr;
    if (!cfg || !out || !gateup_absmax) return MOE_ERR_INVALID_ARG;
    return prepare_impl(cfg, expert_first, n_local, w_gate, w_up, w_down, w_router, act_absmax, gateup_absmax,
                        stream, out);
}

size_t moe_w8a8_ep_dispatch_workspace_size(const moe_w8a8_weights* w, int32_t max_tokens) {
    if (!w || max_tokens < 0) return 0;
    return ws_layout(w, max_tokens, WS_ROUTE).total;
}

size_t moe_w8a8_ep_experts_workspace_size(const moe_w8a8_weights* w, int32_t rows) {
    if (!w || rows < 0) return 0;
    const moe_w8a8_weights v = expert_view(w);
    return ws_layout(&v, rows, WS_EXPERTS).total;
}

moe_status moe_w8a8_ep_dispatch(const moe_w8a8_weights* w, const void* x, int32_t T, const float* router_bias,
                                const float* router_logits, void* send, int32_t* expert_offsets, void* workspace,
                                size_t workspace_bytes, const moe_w8a8_debug* dbg, moe_stream_t stream) {
    if (!w || T < 0 || !expert_offsets) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_config& c = w->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) {
        CUDA_TRY(cudaMemsetAsync(expert_offsets, 0, (size_t)(c.n_experts + 1) * 4, s));
        return MOE_OK;
    }
    if (!x || !send || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign || misaligned16(send) || misaligned16(x) || misaligned16(router_bias) ||
        misaligned16(router_logits))
        return MOE_ERR_INVALID_ARG;
    if (!on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(w, T, WS_ROUTE);
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    Run r(w, L, (char*)workspace, dbg, s);
    r.prof = false;
    MOE_TRY(route_stage(r, x, T, router_bias, router_logits, choose_path(w, T)));
    MOE_TRY(quant_stage(r, x, T, (int8_t*)send, (int64_t)c.d + kEpTrailerBytes, true, c.expert_format));
    CUDA_TRY(cudaMemcpyAsync(expert_offsets, r.at<int32_t>(L.offsets), (size_t)(c.n_experts + 1) * 4,
                             cudaMemcpyDeviceToDevice, s));
    MOE_TRY(debug_stage(r, T, c.top_k, c.n_experts, true, false));
    const_cast<moe_w8a8_weights*>(w)->last_launches = r.launches;
    return MOE_OK;
}

namespace moe {
namespace {

// The expert view of an expert-parallel handle for R received rows; for rows
// in fixed blocks of block_rows rows (0: contiguous rows), a decode-sized
// block (capacity within the fused launch's limit) keeps the fused launch for
// all R rows, most of which are unused slots of the blocks.
moe_w8a8_weights ep_view(const moe_w8a8_weights* w, int R, int block_rows) {
    moe_w8a8_weights v = expert_view(w);
    if (block_rows > 0 && block_rows - 1 <= w->fused_max_rows) v.fused_max_rows = std::max<int64_t>(v.fused_max_rows, R);
    return v;
}

bool ep_ranks(const moe_w8a8_weights* w, const int32_t* rank_first, int32_t world, EpRanks& out) {
    if (!rank_first || world < 1 || world > kEpMaxWorld || rank_first[0] != 0 ||
        rank_first[world] != w->cfg.n_experts)
        return false;
    for (int g = 0; g < world; ++g)
        if (rank_first[g + 1] <= rank_first[g]) return false;
    for (int g = 0; g <= kEpMaxWorld; ++g) out.first[g] = g <= world ? rank_first[g] : w->cfg.n_experts;
    return true;
}

moe_status ep_experts_impl(const moe_w8a8_weights* w, const void* recv, int32_t R, int block_rows, float* o_rows,
                           void* workspace, size_t workspace_bytes, const moe_w8a8_debug* dbg,
                           moe_stream_t stream) {
    if (!recv || !o_rows || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign || misaligned16(recv) || misaligned16(o_rows)) return MOE_ERR_INVALID_ARG;
    if (!on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_weights v = ep_view(w, R, block_rows);
    if (!path_ok(&v, R)) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int path = choose_path(&v, R);
    const WsLayout L = ws_layout(&v, R, WS_EXPERTS);
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = (cudaStream_t)stream;
    Run r(&v, L, (char*)workspace, dbg, s);
    r.prof = false;
    const int d = v.cfg.d;
    const int64_t rb = (int64_t)d + kEpTrailerBytes;
    const uint8_t* rows = (const uint8_t*)recv;
    int32_t* idx = r.at<int32_t>(L.topk_idx);
    int32_t* ts2row = r.at<int32_t>(L.ts2row);
    if (L.fused_words > 0) CUDA_TRY(cudaMemsetAsync(r.at<int32_t>(L.fused_sync), 0, (size_t)L.fused_words * 4, s));
    // each received row is one (token, slot) pair with k = 1 of the local experts
    // (in fixed blocks: headers and unused rows left out)
    CUDA_TRY(launch_ep_read_experts(rows, R, rb, d, block_rows, w->ep_first, w->n_local, idx, w->status, s));
    CUDA_TRY(launch_permute(idx, R, 1, v.cfg.n_experts, -1, r.at<int32_t>(L.hist), r.at<int32_t>(L.offsets),
                            r.at<int32_t>(L.row2ts), ts2row, r.at<int32_t>(L.meta), r.at<int32_t>(L.active),
                            r.at<int32_t>(L.tiles), r.at<int32_t>(L.pairs), s));
    const bool stream_path = path == MOE_PATH_STREAM;
    CUDA_TRY(launch_ep_gather(rows, R, rb, d, stream_path ? nullptr : ts2row,
                              stream_path ? r.at<int8_t>(L.xq) : r.at<int8_t>(L.aq), r.at<float>(L.sx),
                              r.at<float>(L.topk_w), s));
    r.launches += 4;
    MOE_TRY(expert_stage(r, R, path));
    // un-sort: O of received row r to o_rows[r] (k = 1; rows left out get zeros)
    CUDA_TRY(launch_combine(r.at<void>(L.o), v.cfg.out_dtype == MOE_BF16, ts2row, R, 1, d, MOE_F32, o_rows, s));
    ++r.launches;
    MOE_TRY(debug_stage(r, R, 1, v.cfg.n_experts, false, true));
    const_cast<moe_w8a8_weights*>(w)->last_launches = r.launches;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

moe_status moe_w8a8_ep_experts(const moe_w8a8_weights* w, const void* recv, int32_t R, float* o_rows,
                               void* workspace, size_t workspace_bytes, const moe_w8a8_debug* dbg,
                               moe_stream_t stream) {
    if (!w || R < 0) return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    return ep_experts_impl(w, recv, R, 0, o_rows, workspace, workspace_bytes, dbg, stream);
}

int32_t moe_w8a8_ep_block_rows(const moe_w8a8_weights* w, int32_t block_tokens) {
    if (!w || block_tokens < 1 || (int64_t)block_tokens * w->cfg.top_k + 1 > INT32_MAX / 64) return 0;
    return block_tokens * w->cfg.top_k + 1;
}

moe_status moe_w8a8_ep_pack(const moe_w8a8_weights* w, const void* send, const int32_t* expert_offsets,
                            const int32_t* rank_first, int32_t world, int32_t block_tokens, void* blocks,
                            moe_stream_t stream) {
    if (!w) return MOE_ERR_INVALID_ARG;
    const int block_rows = moe_w8a8_ep_block_rows(w, block_tokens);
    EpRanks ranks;
    if (block_rows == 0 || !ep_ranks(w, rank_first, world, ranks)) return MOE_ERR_INVALID_ARG;
    if (!send || !expert_offsets || !blocks || misaligned16(send) || misaligned16(blocks))
        return MOE_ERR_INVALID_ARG;
    if (!on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    CUDA_TRY(launch_ep_pack((const uint8_t*)send, expert_offsets, ranks, world, block_rows,
                            (int64_t)w->cfg.d + kEpTrailerBytes, (uint8_t*)blocks, (cudaStream_t)stream));
    const_cast<moe_w8a8_weights*>(w)->last_launches = 1;
    return MOE_OK;
}

size_t moe_w8a8_ep_experts_blocked_workspace_size(const moe_w8a8_weights* w, int32_t world,
                                                  int32_t block_tokens) {
    if (!w || world < 1 || world > kEpMaxWorld) return 0;
    const int block_rows = moe_w8a8_ep_block_rows(w, block_tokens);
    if (block_rows == 0) return 0;
    const int R = world * block_rows;
    const moe_w8a8_weights v = ep_view(w, R, block_rows);
    return ws_layout(&v, R, WS_EXPERTS).total;
}

moe_status moe_w8a8_ep_experts_blocked(const moe_w8a8_weights* w, const void* blocks, int32_t world,
                                       int32_t block_tokens, float* o_blocks, void* workspace,
                                       size_t workspace_bytes, const moe_w8a8_debug* dbg, moe_stream_t stream) {
    if (!w || world < 1 || world > kEpMaxWorld) return MOE_ERR_INVALID_ARG;
    const int block_rows = moe_w8a8_ep_block_rows(w, block_tokens);
    if (block_rows == 0) return MOE_ERR_INVALID_ARG;
    return ep_experts_impl(w, blocks, world * block_rows, block_rows, o_blocks, workspace, workspace_bytes, dbg,
                           stream);
}

moe_status moe_w8a8_ep_combine_blocked(const moe_w8a8_weights* w, const float* o_blocks, int32_t T,
                                       const int32_t* rank_first, int32_t world, int32_t block_tokens, void* y,
                                       const void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    if (!w || T < 0) return MOE_ERR_INVALID_ARG;
    const int block_rows = moe_w8a8_ep_block_rows(w, block_tokens);
    EpRanks ranks;
    if (block_rows == 0 || !ep_ranks(w, rank_first, world, ranks) || T > block_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y || !o_blocks || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign || misaligned16(o_blocks) || misaligned16(y)) return MOE_ERR_INVALID_ARG;
    if (!on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_config& c = w->cfg;
    const WsLayout L = ws_layout(w, T, WS_ROUTE);
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const int32_t* ts2row = (const int32_t*)((const char*)workspace + L.ts2row);
    const int32_t* offsets = (const int32_t*)((const char*)workspace + L.offsets);
    CUDA_TRY(launch_combine_blocked(o_blocks, ts2row, offsets, ranks, world, block_rows, T, c.top_k, c.d,
                                    c.out_dtype, y, (cudaStream_t)stream));
    const_cast<moe_w8a8_weights*>(w)->last_launches = 1;
    return MOE_OK;
}

moe_status moe_w8a8_ep_combine(const moe_w8a8_weights* w, const float* o_rows, int32_t T, void* y,
                               const void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    if (!w || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y || !o_rows || !workspace) return MOE_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % kAlign || misaligned16(o_rows) || misaligned16(y)) return MOE_ERR_INVALID_ARG;
    if (!on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    const moe_w8a8_config& c = w->cfg;
    const WsLayout L = ws_layout(w, T, WS_ROUTE);
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const int32_t* ts2row = (const int32_t*)((const char*)workspace + L.ts2row);
    CUDA_TRY(launch_combine(o_rows, 0, ts2row, T, c.top_k, c.d, c.out_dtype, y, (cudaStream_t)stream));
    const_cast<moe_w8a8_weights*>(w)->last_launches = 1;
    return MOE_OK;
}

moe_status moe_w8a8_tensor_peak_loop(int32_t expert_format, int64_t mma_per_sm, double* ops_out,
                                     moe_stream_t stream) {
    if (!ops_out) return MOE_ERR_INVALID_ARG;
    *ops_out = 0.0;
    if (expert_format != MOE_FMT_INT8 && expert_format != MOE_FMT_E4M3) return MOE_ERR_INVALID_ARG;
    if (mma_per_sm <= 0 || mma_per_sm > MOE_PEAK_MAX_MMA) return MOE_ERR_INVALID_ARG;
    int dev = -1, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    CUDA_TRY(launch_tc_peak(expert_format, mma_per_sm, sms, (cudaStream_t)stream));
    *ops_out = (double)sms * (double)mma_per_sm * 2.0 * 128.0 * 256.0 * 32.0;
    return MOE_OK;
}

const char* moe_w8a8_stage_name(int32_t stage) {
    static const char* names[MOE_N_STAGES] = {"router", "topk", "permute", "quant",
                                              "gemm1", "requant", "gemm2", "combine"};
    return (stage >= 0 && stage < MOE_N_STAGES) ? names[stage] : "?";
}

int32_t moe_w8a8_last_launch_count(const moe_w8a8_weights* w) { return w ? w->last_launches : 0; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward without any allocation: the scratch is a fixed device array in this
// file.  In host code `g_noalloc_scratch` names a host-side stand-in, not a
// device address, so its device address is looked up once per device (with
// that device current) and only that address is handed to the kernels.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device); nullptr if the lookup fails.
void* noalloc_scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" moe_status moe_w8a8_forward_noalloc(const moe_w8a8_weights* w, const void* x, int32_t T,
                                               const float* router_bias,
                                               const float* router_logits, void* y,
                                               moe_stream_t stream) {
    if (!w || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !y) return MOE_ERR_INVALID_ARG;
    if (misaligned16(x) || misaligned16(y) || misaligned16(router_bias) || misaligned16(router_logits))
        return MOE_ERR_INVALID_ARG;
    if (!holds_all_experts(w) || !on_handle_device(w)) return MOE_ERR_INVALID_ARG;
    if (!path_ok(w, T)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (ws_layout(w, T).total > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = noalloc_scratch_for_current_device();
    if (!scratch) return MOE_ERR_CUDA;
    return forward_impl(w, x, T, router_bias, router_logits, y, (char*)scratch, nullptr,
                        (cudaStream_t)stream);
}
