// Gate, top-k, sort-by-expert and smoothed per-token quantisation.
// ("Day0 adaptation of ultra-large model inference", section 4: gate ->
// sort -> grouped GEMM -> un-sort -> weighted sum, with top-k routing equal to
// the reference including its tie-break; section 2 item 2: capacity factor.
// "MiniMax-M3 W8A8 on K100AI", s3.2 / s6.4: smoothing and per-token INT8.)
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// ---------------------------------------------------------------------------
// Router logits in the stated fp32 order: for each (t, e), partial sum p
// (p = 0..31) is the fma chain over i ascending of x[t][32i+p] W[32i+p][e] from
// +0, and the 32 partials are combined by xor-butterfly 16, 8, 4, 2, 1.
// A block computes 32 tokens x 32 experts.  Lane p of every warp owns partial p
// for a register tile of 8 tokens x 8 experts (16 warps = 4 token groups x 4
// expert groups); X and W_router are staged in shared memory 128 channels at a
// time, laid out [i][p][t] and [i][p][e] with padded rows so that each lane's 8
// tokens (experts) are one conflict-free pair of 16-byte loads.  The token
// index of X is XOR-swizzled on bits 2-4 by (p / 8, i mod 2) so that the
// staging stores (8 consecutive channels of one token per thread) do not pile
// onto one bank; 4-token groups stay contiguous.
// ---------------------------------------------------------------------------
constexpr int kRtT = 32;         // tokens per block
constexpr int kRtE = 32;         // experts per block
constexpr int kRtKC = 128;       // channels per staged chunk (4 steps of i)
constexpr int kRtPad = 36;       // padded row (floats): 16-byte aligned, rows 4 banks apart
constexpr int kRtThreads = 512;

__device__ __forceinline__ int rt_swz(int p, int i) { return ((((p >> 3) & 3) | ((i & 1) << 2)) << 2); }

__global__ void __launch_bounds__(kRtThreads) router_logits_kernel(
    const void* __restrict__ x, int in_dtype, const float* __restrict__ wr, int T, int d, int E,
    float* __restrict__ logits) {
    pdl_wait();
    pdl_trigger();

    __shared__ __align__(16) float xs[kRtKC / 32][32][kRtPad];
    __shared__ __align__(16) float ws[kRtKC / 32][32][kRtPad];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp >> 2, eg = warp & 3;
    const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
    for (int c = 0; c < d; c += kRtKC) {
        // X chunk: 32 tokens x 128 channels, one group of 8 channels per thread
        {
            const int tt = tid >> 4, j0 = (tid & 15) * 8;
            const int t = t0 + tt;
            float v[8];
            if (t < T) {
                load8_act(x, (int64_t)t * d + c + j0, in_dtype, v);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = (j0 + q) >> 5, pp = (j0 + q) & 31;
                xs[i][pp][tt ^ rt_swz(pp, i)] = v[q];
            }
        }
        // W chunk: 128 rows x 32 experts, 16 bytes per thread (two per thread)
        for (int idx = tid; idx < kRtKC * (kRtE / 4); idx += kRtThreads) {
            const int row = idx >> 3, q4 = idx & 7;
            const int e = e0 + 4 * q4;
            const float* src = wr + (int64_t)(c + row) * E;
            float4 v;
            v.x = e + 0 < E ? src[e + 0] : 0.0f;
            v.y = e + 1 < E ? src[e + 1] : 0.0f;
            v.z = e + 2 < E ? src[e + 2] : 0.0f;
            v.w = e + 3 < E ? src[e + 3] : 0.0f;
            *reinterpret_cast<float4*>(&ws[row >> 5][row & 31][4 * q4]) = v;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kRtKC / 32; ++i) {
            const int sw = rt_swz(lane, i);
            const float4 xa = *reinterpret_cast<const float4*>(&xs[i][lane][(tg * 8) ^ sw]);
            const float4 xb = *reinterpret_cast<const float4*>(&xs[i][lane][(tg * 8 + 4) ^ sw]);
            const float4 wa = *reinterpret_cast<const float4*>(&ws[i][lane][eg * 8]);
            const float4 wb = *reinterpret_cast<const float4*>(&ws[i][lane][eg * 8 + 4]);
            const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            float v = acc[a][b];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            acc[a][b] = v;
        }
    // every lane now holds all 64 logits of the warp's tile; lane q writes entries q and q + 32
#pragma unroll
    for (int v = 0; v < 64; ++v) {
        if ((v & 31) != lane) continue;
        const int t = t0 + tg * 8 + (v >> 3), e = e0 + eg * 8 + (v & 7);
        if (t < T && e < E) logits[(int64_t)t * E + e] = acc[v >> 3][v & 7];
    }
}

// Router logits, same order, with the X and W tiles streamed into shared
// memory by cp.async through a 3-stage ring so that global loads overlap the
// FMAs.  X is kept as it arrives ([t][channel], bf16 or fp32); lane p reads its
// 8 tokens' values x[t][32i+p] one element at a time (a warp reads 32
// consecutive channels: conflict-free).  W rows are padded to 36 floats so the
// two 16-byte loads of a lane's 8 experts do not conflict.  Needs E % 4 == 0.
constexpr int kRaStages = 3;
constexpr int kRaWPad = 36;

template <int XB>   // bytes per X element: 2 (bf16) or 4 (fp32)
struct RouterAsyncSmem {
    uint8_t x[kRaStages][kRtT][kRtKC * XB];
    float w[kRaStages][kRtKC][kRaWPad];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int XB>
__global__ void __launch_bounds__(kRtThreads) router_logits_async_kernel(
    const void* __restrict__ x, const float* __restrict__ wr, int T, int d, int E,
    float* __restrict__ logits) {
    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) uint8_t smem_raw[];
    RouterAsyncSmem<XB>& sm = *reinterpret_cast<RouterAsyncSmem<XB>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp >> 2, eg = warp & 3;
    const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
    const int nchunks = d / kRtKC;
    constexpr int kXChunks = kRtT * kRtKC * XB / 16;   // 16-byte pieces of an X tile
    constexpr int kWChunks = kRtKC * kRtE / 4;         // 16-byte pieces of a W tile

    auto issue = [&](int c, int stage) {
        for (int q = tid; q < kXChunks; q += kRtThreads) {
            const int tt = q / (kRtKC * XB / 16), part = q % (kRtKC * XB / 16);
            const int t = t0 + tt;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(x) +
                                 ((int64_t)min(t, T - 1) * d + (int64_t)c * kRtKC) * XB + part * 16;
            cp_async16(&sm.x[stage][tt][part * 16], src, t < T ? 16 : 0);
        }
        for (int q = tid; q < kWChunks; q += kRtThreads) {
            const int row = q / (kRtE / 4), c4 = q % (kRtE / 4);
            const int e = e0 + 4 * c4;
            const float* src = wr + (int64_t)(c * kRtKC + row) * E + min(e, E - 4);
            cp_async16(&sm.w[stage][row][4 * c4], src, e < E ? 16 : 0);
        }
        cp_async_commit();
    };

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

    issue(0, 0);
    if (nchunks > 1) issue(1, 1); else cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<1>();
        __syncthreads();
        if (c + 2 < nchunks) issue(c + 2, (c + 2) % kRaStages); else cp_async_commit();
        const int st = c % kRaStages;
#pragma unroll
        for (int i = 0; i < kRtKC / 32; ++i) {
            float xv[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const uint8_t* px = &sm.x[st][tg * 8 + a][(32 * i + lane) * XB];
                xv[a] = XB == 2 ? bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(px))
                                : *reinterpret_cast<const float*>(px);
            }
            const float4 wa = *reinterpret_cast<const float4*>(&sm.w[st][32 * i + lane][eg * 8]);
            const float4 wb = *reinterpret_cast<const float4*>(&sm.w[st][32 * i + lane][eg * 8 + 4]);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            float v = acc[a][b];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            acc[a][b] = v;
        }
#pragma unroll
    for (int v = 0; v < 64; ++v) {
        if ((v & 31) != lane) continue;
        const int t = t0 + tg * 8 + (v >> 3), e = e0 + eg * 8 + (v & 7);
        if (t < T && e < E) logits[(int64_t)t * E + e] = acc[v >> 3][v & 7];
    }
}

// Router logits for bf16 X and E % 32 == 0, same fixed order, with a larger
// register tile: each lane keeps its chain position for 16 tokens x 8 experts
// (128 accumulators), so every W value it reads from shared memory feeds 16
// FMAs and every X value 8.  256 threads: warp w covers tokens (w >> 2) * 16
// and experts (w & 3) * 8 of the block's 32 x 32 tile.  X ([token][channel],
// rows padded by 16 bytes) and W (rows padded to 36 floats, so a quarter
// warp's 16-byte loads hit distinct banks) arrive by cp.async through a
// 3-stage ring of 256-channel chunks; a lane reads its 16 tokens' values of
// channel 32i + lane one bf16 at a time (a warp reads 64 consecutive bytes).
// Measured against transposed-X and 128-channel variants of the same tile
// (identical logits): this one was the fastest, by 5%.
constexpr int kRwThreads = 256;
constexpr int kRwKC = 256;        // channels per staged chunk (8 steps of i)

struct RouterWideSmem {
    uint16_t x[kRaStages][kRtT][kRwKC + 8];
    float w[kRaStages][kRwKC][kRaWPad];
};

__global__ void __launch_bounds__(kRwThreads, 1) router_logits_wide_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ wr, int T, int d, int E,
    float* __restrict__ logits) {
    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) uint8_t smem_raw[];
    RouterWideSmem& sm = *reinterpret_cast<RouterWideSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp >> 2, eg = warp & 3;
    const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
    const int nchunks = d / kRwKC;

    auto issue = [&](int c, int stage) {
        for (int q = tid; q < kRtT * kRwKC / 8; q += kRwThreads) {
            const int tt = q / (kRwKC / 8), part = q % (kRwKC / 8);
            cp_async16(&sm.x[stage][tt][part * 8], x + (int64_t)min(t0 + tt, T - 1) * d + (int64_t)c * kRwKC + part * 8,
                       16);
        }
        for (int q = tid; q < kRwKC * kRtE / 4; q += kRwThreads) {
            const int row = q / (kRtE / 4), c4 = q % (kRtE / 4);
            cp_async16(&sm.w[stage][row][4 * c4], wr + (int64_t)(c * kRwKC + row) * E + e0 + 4 * c4, 16);
        }
        cp_async_commit();
    };

    float acc[16][8];
#pragma unroll
    for (int a = 0; a < 16; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

    issue(0, 0);
    if (nchunks > 1) issue(1, 1); else cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<1>();
        __syncthreads();
        if (c + 2 < nchunks) issue(c + 2, (c + 2) % kRaStages); else cp_async_commit();
        const int st = c % kRaStages;
#pragma unroll
        for (int i = 0; i < kRwKC / 32; ++i) {
            const int k = 32 * i + lane;
            float xv[16];
#pragma unroll
            for (int a = 0; a < 16; ++a) xv[a] = __uint_as_float((uint32_t)sm.x[st][tg * 16 + a][k] << 16);
            const float4 wa = *reinterpret_cast<const float4*>(&sm.w[st][k][eg * 8]);
            const float4 wb = *reinterpret_cast<const float4*>(&sm.w[st][k][eg * 8 + 4]);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int a = 0; a < 16; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int a = 0; a < 16; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            float v = acc[a][b];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            acc[a][b] = v;
        }
    // every lane holds all 128 logits of the warp's tile; lane q writes entries q, q+32, q+64, q+96
#pragma unroll
    for (int v = 0; v < 128; ++v) {
        if ((v & 31) != lane) continue;
        const int t = t0 + tg * 16 + (v >> 3), e = e0 + eg * 8 + (v & 7);
        if (t < T) logits[(int64_t)t * E + e] = acc[v >> 3][v & 7];
    }
}

// ---------------------------------------------------------------------------
// Top-k + gate weights, one warp per token.  l_e = logit + bias_e; k rounds of
// a warp argmax on (l descending, e ascending); w = softmax of the selected
// logits (renormalised) with the layer's exp, sum in slot order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool better(float v, int i, float v2, int i2) {
    return v > v2 || (v == v2 && i < i2);
}

// One warp: top-k and gate weights of token t.  lsh: kMaxE floats of shared
// scratch for this warp (used when the softmax runs over all E experts).
// When idx_copy is given, the chosen experts are also written there.
__device__ __forceinline__ void topk_token(const float* __restrict__ logits,
                                           const float* __restrict__ bias, int t, int E, int k,
                                           int renorm, int32_t* __restrict__ idx,
                                           float* __restrict__ wts, float* __restrict__ logits_out,
                                           float* lsh, int32_t* idx_copy, int lane) {
    constexpr int kPer = kMaxE / 32;
    float l[kPer];
    bool taken[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        float v = -INFINITY;
        if (e < E) {
            v = logits[(int64_t)t * E + e];
            if (bias) v = __fadd_rn(v, bias[e]);
            if (logits_out) logits_out[(int64_t)t * E + e] = v;
            lsh[e] = v;
        }
        l[m] = v;
        taken[m] = e >= E;
    }
    float sel_v[kMaxK];
    int sel_i[kMaxK];
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) {
        if (s >= k) break;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int e = lane + 32 * m;
            if (!taken[m] && better(l[m], e, bv, bi)) { bv = l[m]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m)
            if (lane + 32 * m == bi) taken[m] = true;
        sel_v[s] = bv;
        sel_i[s] = bi;
    }
    __syncwarp();
    // slot s is handled by lane s: exp of each selected logit in parallel, the
    // normaliser summed in slot (or expert) order by a fixed sequence of adds
    const float lmax = sel_v[0];
    float z = 0.0f;
    if (renorm) {
        for (int s = 0; s < k; ++s) z = __fadd_rn(z, moe_exp(__fsub_rn(sel_v[s], lmax)));
    } else {
        for (int e = 0; e < E; ++e) z = __fadd_rn(z, moe_exp(__fsub_rn(lsh[e], lmax)));
    }
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) {
        if (s >= k) break;
        if (lane == s) {
            idx[(int64_t)t * k + s] = sel_i[s];
            wts[(int64_t)t * k + s] = __fdiv_rn(moe_exp(__fsub_rn(sel_v[s], lmax)), z);
            if (idx_copy) idx_copy[t * k + s] = sel_i[s];
        }
    }
}

__global__ void topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T,
                            int E, int k, int renorm, int32_t* __restrict__ idx,
                            float* __restrict__ wts, float* __restrict__ logits_out) {
    pdl_wait();
    pdl_trigger();

    __shared__ float lsh[8][kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    topk_token(logits, bias, t, E, k, renorm, idx, wts, logits_out, lsh[warp], nullptr, lane);
}

// ---------------------------------------------------------------------------
// Certified router, second step (the first is router_tc_kernel: approximate
// logits l~ from the tensor cores).  One warp per token:
//   S = sum_j |x_j| max_e |W_g[j][e]|  bounds sum_j |x_j| |W_g[j][e]| for every e;
//   a_e = l~_e + bias_e; v_k = the k-th largest a_e;
//   B = c_err S + 2^-22 (max_e |a_e| + 1) bounds |a_e - l_e| for every e, l_e
//       being the logit in the stated fp32 order (+ bias): c_err covers the bf16
//       split of W_g (2^-16), the fp32 order's own rounding and the tensor
//       cores' fp32 accumulation (modelled as at most 2^-21 of the running
//       absolute sum per MMA step); the last term the two bias additions;
//   candidates C = { e : a_e >= v_k - 2B }.
// An expert outside C has l_e < v_k - B <= l_j for each of the k experts j with
// the largest a_j, so it cannot be among the top k: the top k of the exact
// logits over C alone is the top k over all experts, ties included.  The
// candidates' logits are computed in the stated order (lane chains, xor
// butterfly, then + bias), the others set to -inf, and topk_token chooses and
// weighs exactly as for fully computed logits.  logits_out (debug) receives
// exact logits for candidates and a_e for the rest.
// ---------------------------------------------------------------------------
constexpr int kSelWarps = 4;
constexpr int kSelCand = 4;   // candidates evaluated together (more: further passes)
constexpr int kSelJ = 2;      // 16-byte steps of every candidate loaded together (with 5 blocks
                              // per SM: 96 registers, 20 warps; faster than 4 steps at 16 warps)

// W_g and max|W_g| are stored lane-interleaved: element j = 32 i + p (lane p,
// step i) of a row sits at [i / 4][p][i % 4], so lane p reads its 4 steps
// 4j..4j+3 with one 16-byte load and a warp reads 512 contiguous bytes.
__device__ __forceinline__ float4 ld_lane4(const float* rowbase, int j, int lane) {
    return __ldg(reinterpret_cast<const float4*>(rowbase) + (int64_t)j * 32 + lane);
}

__global__ void __launch_bounds__(kSelWarps * 32, 5) router_select_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ approx, const float* __restrict__ bias,
    const float* __restrict__ wt, const float* __restrict__ wmax, int T, int d, int E, int k, float c_err,
    float* __restrict__ sel, int32_t* __restrict__ idx, float* __restrict__ wts, float* __restrict__ logits_out) {
    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw) + (size_t)warp * d;   // this warp's token row
    float* lsh = reinterpret_cast<float*>(smem_raw + (size_t)kSelWarps * d * 2) + warp * kMaxE;
    const int t = blockIdx.x * kSelWarps + warp;
    if (t >= T) return;
    {
        // the token's X row into shared memory: every 16-byte piece in flight at once
        const uint16_t* src = x + (int64_t)t * d;
        for (int i = lane; i < d / 8; i += 32) cp_async16(xs + 8 * i, src + 8 * i, 16);
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
    }
    const int nj = d / 128;   // 16-byte steps per lane
    float S = 0.0f;
#pragma unroll 8
    for (int j = 0; j < nj; ++j) {
        const float4 m4 = ld_lane4(wmax, j, lane);
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) S = fmaf(fabsf(bf16_bits_to_f32(xs[32 * (4 * j + q) + lane])), mv[q], S);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    constexpr int kPer = kMaxE / 32;
    float a[kPer], ex[kPer];
    bool taken[kPer];
    float amax = 0.0f;
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        a[m] = -INFINITY;
        ex[m] = -INFINITY;
        if (e < E) {
            float v = approx[(int64_t)t * E + e];
            if (bias) v = __fadd_rn(v, bias[e]);
            a[m] = v;
            amax = fmaxf(amax, fabsf(v));
        }
        taken[m] = e >= E;
    }
    amax = warp_max(amax);
    float vk = 0.0f;
    for (int s = 0; s < k; ++s) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int e = lane + 32 * m;
            if (!taken[m] && better(a[m], e, bv, bi)) { bv = a[m]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m)
            if (lane + 32 * m == bi) taken[m] = true;
        vk = bv;
    }
    const float B = c_err * S * (1.0f + 0x1p-10f) + 0x1p-22f * (amax + 1.0f);
    const float thr = vk - 2.0f * B * (1.0f + 0x1p-10f);
    unsigned cmask[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) cmask[m] = __ballot_sync(0xffffffffu, lane + 32 * m < E && a[m] >= thr);
    // candidates in passes of kSelCand: all their chains advance together
    int m0 = 0;
    while (true) {
        int ce[kSelCand];
        int nc = 0;
        for (; m0 < kPer && nc < kSelCand; ) {
            if (cmask[m0] == 0u) { ++m0; continue; }
            const int b = __ffs(cmask[m0]) - 1;
            cmask[m0] &= cmask[m0] - 1;
            ce[nc++] = b + 32 * m0;
        }
        if (nc == 0) break;
        float acc[kSelCand];
#pragma unroll
        for (int c = 0; c < kSelCand; ++c) acc[c] = 0.0f;
        for (int j0 = 0; j0 < nj; j0 += kSelJ) {
            // all loads of kSelJ steps of every candidate first (one L2 round trip), then the
            // FMAs, each chain in its own channel order
            float4 w4[kSelJ][kSelCand];
#pragma unroll
            for (int jj = 0; jj < kSelJ; ++jj)
#pragma unroll
                for (int c = 0; c < kSelCand; ++c)
                    if (c < nc && j0 + jj < nj) w4[jj][c] = ld_lane4(wt + (int64_t)ce[c] * d, j0 + jj, lane);
#pragma unroll
            for (int jj = 0; jj < kSelJ; ++jj) {
                if (j0 + jj >= nj) break;
                float xv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[q] = bf16_bits_to_f32(xs[32 * (4 * (j0 + jj) + q) + lane]);
#pragma unroll
                for (int c = 0; c < kSelCand; ++c) {
                    if (c < nc) {
                        acc[c] = __fmaf_rn(xv[0], w4[jj][c].x, acc[c]);
                        acc[c] = __fmaf_rn(xv[1], w4[jj][c].y, acc[c]);
                        acc[c] = __fmaf_rn(xv[2], w4[jj][c].z, acc[c]);
                        acc[c] = __fmaf_rn(xv[3], w4[jj][c].w, acc[c]);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kSelCand; ++c) {
            if (c < nc) {
                float v = acc[c];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (bias) v = __fadd_rn(v, bias[ce[c]]);
#pragma unroll
                for (int m = 0; m < kPer; ++m)
                    if (ce[c] == lane + 32 * m) ex[m] = v;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        if (e < E) {
            const bool cand = a[m] >= thr;
            sel[(int64_t)t * E + e] = cand ? ex[m] : -INFINITY;
            if (logits_out) logits_out[(int64_t)t * E + e] = cand ? ex[m] : a[m];
        }
    }
    __syncwarp();
    topk_token(sel, nullptr, t, E, k, 1, idx, wts, nullptr, lsh, nullptr, lane);
}

// ---------------------------------------------------------------------------
// Sort by expert.  Entry i (= t*k + slot) of expert e gets position
// pos = #(earlier entries of e) and is kept when pos < capacity; kept rows are
// ordered by expert, then by i.  Large inputs: a histogram per chunk of
// kPermChunk entries, then a scatter in which every block derives the global
// expert offsets and its own prefix from the histogram.  Small inputs: one
// block does top-k, histogram, scan and scatter.
// ---------------------------------------------------------------------------

// Expert offsets (exclusive scan of kept counts) and the lists the expert
// kernels read: active experts, 128-row tiles and 256-row pair tiles (for the
// kernels that run one 256-row MMA on a pair of SMs).  Run by one full warp:
// lane l owns experts [l*per, l*per + per), exclusive warp scans place its
// offsets, active entries, tiles and pair tiles.
__device__ void write_offsets_and_lists(const int* kept, int E, int* off, int32_t* offsets,
                                        int32_t* meta, int32_t* active, int32_t* tiles, int32_t* pairs,
                                        int lane) {
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int rows = 0, nact = 0, ntl = 0, npr = 0;
    for (int e = e0; e < e1; ++e) {
        rows += kept[e];
        nact += kept[e] > 0;
        ntl += (kept[e] + kTileM - 1) / kTileM;
        npr += (kept[e] + kPairM - 1) / kPairM;
    }
    int xr = rows, xa = nact, xt = ntl, xp = npr;   // inclusive scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, xr, o);
        const int b = __shfl_up_sync(0xffffffffu, xa, o);
        const int c = __shfl_up_sync(0xffffffffu, xt, o);
        const int d = __shfl_up_sync(0xffffffffu, xp, o);
        if (lane >= o) { xr += a; xa += b; xt += c; xp += d; }
    }
    int r = xr - rows, na = xa - nact, nt = xt - ntl, np = xp - npr;
    for (int e = e0; e < e1; ++e) {
        off[e] = r;
        offsets[e] = r;
        if (kept[e] > 0) active[na++] = e;
        for (int m = 0; m * kTileM < kept[e]; ++m) {
            tiles[2 * nt] = e;
            tiles[2 * nt + 1] = r + m * kTileM;
            ++nt;
        }
        for (int m = 0; m * kPairM < kept[e]; ++m) {
            pairs[2 * np] = e;
            pairs[2 * np + 1] = r + m * kPairM;
            ++np;
        }
        r += kept[e];
    }
    if (lane == 31) {
        off[E] = xr;
        offsets[E] = xr;
        meta[META_R] = xr;
        meta[META_NACTIVE] = xa;
        meta[META_NTILES] = xt;
        meta[META_NPAIRS] = xp;
    }
}

// Stable ranks of entries [base, base + len) in rounds of blockDim.x: warp
// match for ranks inside a warp, per-warp counts (wcnt, [warps][kMaxE]) for
// ranks across warps, running per-expert totals across rounds.  pre[e]: entries
// of e before `base`.  Block-wide; needs off[], pre[], running[] in shared.
__device__ void scatter_entries(const int32_t* idx, int base, int len, int E, int cap,
                                const int* pre, const int* off, int* running, int (*wcnt)[kMaxE],
                                int32_t* __restrict__ row2ts, int32_t* __restrict__ ts2row) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    for (int r0 = 0; r0 < len; r0 += blockDim.x) {
        for (int i = tid; i < nw * E; i += blockDim.x) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int i = base + r0 + tid;
        const bool in = r0 + tid < len;
        const int e = in ? idx[i] : -1;
        const bool valid = in && e >= 0;   // e < 0: an entry to leave out (no row)
        const unsigned m = __match_any_sync(0xffffffffu, e);
        const int rank_w = __popc(m & ((1u << lane) - 1u));
        if (valid && rank_w == 0) wcnt[warp][e] = __popc(m);
        __syncthreads();
        if (in && !valid) ts2row[i] = -1;
        if (valid) {
            int rank = running[e] + rank_w;
            for (int w2 = 0; w2 < warp; ++w2) rank += wcnt[w2][e];
            const int pos = pre[e] + rank;
            const int row = off[e] + pos;
            if ((cap < 0 || pos < cap) && row < off[E]) {   // row < R always holds; guard the store
                ts2row[i] = row;
                row2ts[row] = i;
            } else {
                ts2row[i] = -1;
            }
        }
        __syncthreads();
        for (int e2 = tid; e2 < E; e2 += blockDim.x) {
            int s = 0;
            for (int w2 = 0; w2 < nw; ++w2) s += wcnt[w2][e2];
            running[e2] += s;
        }
        __syncthreads();
    }
}

__global__ void perm_hist_kernel(const int32_t* __restrict__ idx, int n, int E,
                                 int32_t* __restrict__ hist) {
    pdl_wait();
    pdl_trigger();

    __shared__ int cnt[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int base = blockIdx.x * kPermChunk;
    for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x)
        if (base + i < n) {
            const int e = idx[base + i];
            if (e >= 0) atomicAdd(&cnt[e], 1);   // e < 0: an entry to leave out
        }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = cnt[e];
}

constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads) perm_scatter_kernel(
    const int32_t* __restrict__ idx, int n, int E, int cap, int nblk,
    const int32_t* __restrict__ hist, int32_t* __restrict__ offsets, int32_t* __restrict__ row2ts,
    int32_t* __restrict__ ts2row, int32_t* __restrict__ meta, int32_t* __restrict__ active,
    int32_t* __restrict__ tiles, int32_t* __restrict__ pairs, int32_t* __restrict__ zero_words, int n_zero) {
    pdl_wait();
    pdl_trigger();
    // counters a later kernel of this forward starts from zero (the fused expert launch)
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0;

    __shared__ int pre[kMaxE], off[kMaxE + 1], running[kMaxE], kept[kMaxE];
    __shared__ int wcnt[kPermThreads / 32][kMaxE];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        int tot = 0, before = 0;
        for (int b = 0; b < nblk; ++b) {
            const int h = hist[(int64_t)b * E + e];
            tot += h;
            if (b < (int)blockIdx.x) before += h;
        }
        pre[e] = before;
        kept[e] = cap < 0 ? tot : min(tot, cap);
        running[e] = 0;
    }
    __syncthreads();
    if (tid < 32) {
        if (blockIdx.x == 0) {
            write_offsets_and_lists(kept, E, off, offsets, meta, active, tiles, pairs, tid);
        } else if (tid == 0) {
            int acc = 0;
            for (int e = 0; e < E; ++e) { off[e] = acc; acc += kept[e]; }
            off[E] = acc;
        }
    }
    __syncthreads();
    const int base = blockIdx.x * kPermChunk;
    scatter_entries(idx, base, min(kPermChunk, n - base), E, cap, pre, off, running, wcnt, row2ts,
                    ts2row);
}

// Small inputs (T*k <= kRouteSmallMax): top-k, histogram, scan and stable
// scatter in one block of 1024 threads (warp w does tokens w, w + 32, ...).
constexpr int kRouteSmallThreads = 1024;
constexpr int kRouteSmallMax = 2048;

struct RouteSmallSmem {
    int32_t idx[kRouteSmallMax];
    int pre[kMaxE], off[kMaxE + 1], running[kMaxE], kept[kMaxE];
    union {
        float lsh[kRouteSmallThreads / 32][kMaxE];
        int wcnt[kRouteSmallThreads / 32][kMaxE];
    } u;
};

__global__ void __launch_bounds__(kRouteSmallThreads) route_small_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
    int renorm, int cap, int32_t* __restrict__ idx, float* __restrict__ wts,
    float* __restrict__ logits_out, int32_t* __restrict__ offsets, int32_t* __restrict__ row2ts,
    int32_t* __restrict__ ts2row, int32_t* __restrict__ meta, int32_t* __restrict__ active,
    int32_t* __restrict__ tiles, int32_t* __restrict__ pairs, int32_t* __restrict__ zero_words, int n_zero) {
    pdl_wait();
    pdl_trigger();
    // counters a later kernel of this forward starts from zero (the fused expert launch)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0;

    extern __shared__ __align__(16) uint8_t smem_raw[];
    RouteSmallSmem& sm = *reinterpret_cast<RouteSmallSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = T * k;
    for (int t = warp; t < T; t += kRouteSmallThreads / 32)
        topk_token(logits, bias, t, E, k, renorm, idx, wts, logits_out, sm.u.lsh[warp], sm.idx, lane);
    for (int e = tid; e < E; e += blockDim.x) {
        sm.kept[e] = 0;
        sm.pre[e] = 0;
        sm.running[e] = 0;
    }
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) atomicAdd(&sm.kept[sm.idx[i]], 1);
    __syncthreads();
    if (cap >= 0)
        for (int e = tid; e < E; e += blockDim.x) sm.kept[e] = min(sm.kept[e], cap);
    __syncthreads();
    if (tid < 32) write_offsets_and_lists(sm.kept, E, sm.off, offsets, meta, active, tiles, pairs, tid);
    __syncthreads();
    scatter_entries(sm.idx, 0, n, E, cap, sm.pre, sm.off, sm.running, sm.u.wcnt, row2ts, ts2row);
}

// ---------------------------------------------------------------------------
// Smoothed per-token quantisation: x' = fp32(x * inv_s); sx = amax/127;
// q = rint(x'/sx) clamped to +-127.  One block per token; each thread owns
// groups of 8 channels.  Writes xq[t] (unless xq is null) and, when aq is
// given, the copy of the token's codes into every kept (t, slot) row of the
// expert-sorted matrix.
// ---------------------------------------------------------------------------
// One block of kSqThreads threads per token: thread i owns channel groups i,
// i + kSqThreads, ... (8 channels each); all of a thread's loads are issued before the block
// max (one shared-memory exchange), then the codes are written to xq[t] and,
// for the tensor-core path, to every kept (t, slot) row of the sorted copy.

template <int kSqMaxGroups, int FMT, int kSqThreads>   // groups of 8 channels per thread: d <= kSqThreads x 8 x kSqMaxGroups
__global__ void __launch_bounds__(kSqThreads) smooth_quant_kernel(
    const void* __restrict__ x, int in_dtype, const float* __restrict__ inv_s, float act_clip, int T, int d,
    int k, const int32_t* __restrict__ ts2row, int8_t* __restrict__ xq, float* __restrict__ sx,
    int8_t* __restrict__ aq, int64_t aq_ld, const float* __restrict__ wts, const int32_t* __restrict__ idx) {
    // X is an input of the forward and xq / sx are read only by later kernels of
    // this forward: when this kernel starts (its predecessor has passed its own
    // wait) every kernel of the previous forward has finished, so the codes are
    // formed while the routing kernel still runs; only the copy into the
    // expert-sorted rows waits for the routing (ts2row).
    pdl_trigger();

    __shared__ float red[kSqThreads / 32];
    const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int ng = d / 8;
    float v[kSqMaxGroups][8];
#pragma unroll
    for (int gi = 0; gi < kSqMaxGroups; ++gi) {
        const int g = tid + kSqThreads * gi;
        if (g < ng) load8_act(x, (int64_t)t * d + g * 8, in_dtype, v[gi]);
    }
    float m = 0.0f;
#pragma unroll
    for (int gi = 0; gi < kSqMaxGroups; ++gi) {
        const int g = tid + kSqThreads * gi;
        if (g < ng) {
            const float4 s0 = *reinterpret_cast<const float4*>(inv_s + g * 8);
            const float4 s1 = *reinterpret_cast<const float4*>(inv_s + g * 8 + 4);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                v[gi][c] = __fmul_rn(v[gi][c], sv[c]);
                m = fmaxf(m, fabsf(v[gi][c]));
            }
        }
    }
    m = warp_max(m);
    if (lane == 0) red[tid >> 5] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kSqThreads / 32; ++w) m = fmaxf(m, red[w]);
    if (act_clip > 0.0f) m = fminf(m, act_clip);   // saturating clip: values beyond it go to +-127
    const float s = m > 0.0f ? __fdiv_rn(m, fmt_qmax<FMT>()) : 0.0f;
    const float rs = s > 0.0f ? __frcp_rn(s) : 0.0f;
    if (tid == 0) sx[t] = s;
    uint2 packed[kSqMaxGroups];
#pragma unroll
    for (int gi = 0; gi < kSqMaxGroups; ++gi) {
        const int g = tid + kSqThreads * gi;
        if (g >= ng) continue;
        packed[gi] = s > 0.0f ? make_uint2(fmt_codes4<FMT>(v[gi][0], v[gi][1], v[gi][2], v[gi][3], s, rs),
                                           fmt_codes4<FMT>(v[gi][4], v[gi][5], v[gi][6], v[gi][7], s, rs))
                              : make_uint2(0u, 0u);
        if (xq) *reinterpret_cast<uint2*>(xq + (int64_t)t * d + g * 8) = packed[gi];
    }
    pdl_wait();   // the routing of this forward is complete from here on
    if (!aq) return;
    int rows[kMaxK];
#pragma unroll
    for (int sl = 0; sl < kMaxK; ++sl) rows[sl] = sl < k ? ts2row[(int64_t)t * k + sl] : -1;
#pragma unroll
    for (int gi = 0; gi < kSqMaxGroups; ++gi) {
        const int g = tid + kSqThreads * gi;
        if (g >= ng) continue;
#pragma unroll
        for (int sl = 0; sl < kMaxK; ++sl)
            if (rows[sl] >= 0) *reinterpret_cast<uint2*>(aq + (int64_t)rows[sl] * aq_ld + g * 8) = packed[gi];
    }
    if (wts && tid < k) {   // expert-parallel send rows: the trailer after the codes
        const int64_t ts = (int64_t)t * k + tid;
        const int row = ts2row[ts];
        if (row >= 0)
            *reinterpret_cast<int4*>(aq + (int64_t)row * aq_ld + d) =
                make_int4(__float_as_int(s), __float_as_int(wts[ts]), idx[ts], (int)ts);
    }
}

// Expert-parallel receive side: the local expert of each received row.  In
// fixed blocks (block_rows > 0) row 0 of each block of block_rows rows is the
// block's header (its first word the number of rows that follow) and rows
// past that number are left out (idx -1).
__global__ void ep_read_experts_kernel(const uint8_t* __restrict__ recv, int R, int64_t row_bytes, int d,
                                       int block_rows, int ep_first, int n_local, int32_t* __restrict__ idx,
                                       int32_t* __restrict__ status) {
    pdl_wait();
    pdl_trigger();
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    if (block_rows > 0) {
        const int g = r / block_rows, i = r % block_rows;
        int count = *reinterpret_cast<const int32_t*>(recv + (int64_t)g * block_rows * row_bytes);
        if (count < 0 || count > block_rows - 1) {
            if (i == 0 && atomicCAS(status, 0, (int32_t)MOE_ERR_INVALID_ARG) == 0) {
                status[1] = kSiteEpBlock;
                status[2] = g;
                status[3] = count;
            }
            count = 0;
        }
        if (i == 0 || i > count) {
            idx[r] = -1;
            return;
        }
    }
    const EpTrailer* tr = reinterpret_cast<const EpTrailer*>(recv + (int64_t)r * row_bytes + d);
    const int e = tr->expert - ep_first;
    if (e < 0 || e >= n_local) {
        if (atomicCAS(status, 0, (int32_t)MOE_ERR_INVALID_ARG) == 0) {
            status[1] = kSiteEpExpert;
            status[2] = r;
            status[3] = tr->expert;
        }
        idx[r] = 0;
        return;
    }
    idx[r] = e;
}

// Codes of each received row to its sorted row (or row r), scale and gate
// weight to sx[r], wts[r]: one warp per row, 16-byte copies.
constexpr int kEpGatherWarps = 8;
__global__ void __launch_bounds__(kEpGatherWarps * 32) ep_gather_kernel(
    const uint8_t* __restrict__ recv, int R, int64_t row_bytes, int d, const int32_t* __restrict__ ts2row,
    int8_t* __restrict__ dst, float* __restrict__ sx, float* __restrict__ wts) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * kEpGatherWarps + (threadIdx.x >> 5);
    if (r >= R) return;
    const uint8_t* src = recv + (int64_t)r * row_bytes;
    const int64_t drow = ts2row ? ts2row[r] : r;
    if (drow < 0) return;   // a row left out (a fixed block's header or unused row)
    int8_t* out = dst + drow * d;
    for (int j = lane * 16; j < d; j += 32 * 16)
        *reinterpret_cast<int4*>(out + j) = *reinterpret_cast<const int4*>(src + j);
    if (lane == 0) {
        const EpTrailer* tr = reinterpret_cast<const EpTrailer*>(src + d);
        sx[r] = tr->sx;
        wts[r] = tr->w;
    }
}

// Fixed-block send buffer: block g (of `block_rows` rows) holds a header row
// (first word: the number of rows for rank g's experts, the rest zero) and
// then those rows, copied from the expert-major send rows
// [offsets[first[g]], offsets[first[g + 1]]).  One warp per block row,
// 16-byte copies; rows past the count are not written.
__global__ void __launch_bounds__(kEpGatherWarps * 32) ep_pack_kernel(
    const uint8_t* __restrict__ send, const int32_t* __restrict__ offsets, EpRanks ranks, int block_rows,
    int64_t row_bytes, uint8_t* __restrict__ blocks) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.y;
    const int i = blockIdx.x * kEpGatherWarps + (threadIdx.x >> 5);
    if (i >= block_rows) return;
    const int lo = offsets[ranks.first[g]], hi = offsets[ranks.first[g + 1]];
    uint8_t* dst = blocks + ((int64_t)g * block_rows + i) * row_bytes;
    if (i == 0) {
        for (int64_t j = lane * 16; j < row_bytes; j += 32 * 16)
            *reinterpret_cast<int4*>(dst + j) = make_int4(j == 0 ? hi - lo : 0, 0, 0, 0);
        return;
    }
    const int r = lo + i - 1;
    if (r >= hi) return;
    const uint8_t* src = send + (int64_t)r * row_bytes;
    for (int64_t j = lane * 16; j < row_bytes; j += 32 * 16)
        *reinterpret_cast<int4*>(dst + j) = *reinterpret_cast<const int4*>(src + j);
}

}  // namespace

cudaError_t launch_router_logits(const void* x, int in_dtype, const float* wr, int T, int d, int E,
                                 float* logits, cudaStream_t s) {
    dim3 grid((T + kRtT - 1) / kRtT, (E + kRtE - 1) / kRtE);
    if (in_dtype == MOE_BF16 && E % kRtE == 0 && d % kRwKC == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
        static std::atomic<uint64_t> wide_attr{0};
        cudaError_t e = smem_attr_once(router_logits_wide_kernel, sizeof(RouterWideSmem), wide_attr);
        if (e != cudaSuccess) return e;
        return launch_pdl(router_logits_wide_kernel, grid, dim3(kRwThreads), sizeof(RouterWideSmem), s,
                          reinterpret_cast<const uint16_t*>(x), wr, T, d, E, logits);
    }
    if (E % 4 == 0 && E >= 4) {
        static std::atomic<uint64_t> attr2{0}, attr4{0};
        cudaError_t e = in_dtype == MOE_BF16
                            ? smem_attr_once(router_logits_async_kernel<2>, sizeof(RouterAsyncSmem<2>), attr2)
                            : smem_attr_once(router_logits_async_kernel<4>, sizeof(RouterAsyncSmem<4>), attr4);
        if (e != cudaSuccess) return e;
        if (in_dtype == MOE_BF16)
            return launch_pdl(router_logits_async_kernel<2>, grid, dim3(kRtThreads), sizeof(RouterAsyncSmem<2>), s,
                              x, wr, T, d, E, logits);
        else
            return launch_pdl(router_logits_async_kernel<4>, grid, dim3(kRtThreads), sizeof(RouterAsyncSmem<4>), s,
                              x, wr, T, d, E, logits);
    } else {
        return launch_pdl(router_logits_kernel, grid, dim3(kRtThreads), 0, s, x, in_dtype, wr, T, d, E, logits);
    }
    return cudaGetLastError();
}

cudaError_t launch_router_select(const moe_w8a8_weights* w, const void* x, int T, const float* approx,
                                 const float* bias, float* sel, int32_t* idx, float* wts, float* logits_out,
                                 cudaStream_t s) {
    const int d = w->cfg.d;
    // bf16 split of W_g (2^-16), the stated order's own rounding ((d/32 + 6) ulps), the
    // tensor cores' accumulation: 2 x (d/16 + 1) MMA steps, 2^-21 of the running sum each
    const double c_err = std::ldexp(1.0, -16) + (d / 32 + 6) * std::ldexp(1.0, -24) +
                         (2.0 * (d / 16) + 2.0) * std::ldexp(1.0, -21);
    const size_t smem = (size_t)kSelWarps * d * 2 + (size_t)kSelWarps * kMaxE * 4;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(router_select_kernel, (size_t)kSelWarps * 16384 * 2 + (size_t)kSelWarps * kMaxE * 4,
                                   attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_select_kernel, dim3((T + kSelWarps - 1) / kSelWarps), dim3(kSelWarps * 32), smem, s,
                      reinterpret_cast<const uint16_t*>(x), approx, bias, w->rt_wt, w->rt_wmax, T, d,
                      w->cfg.n_experts, w->cfg.top_k, (float)c_err, sel, idx, wts, logits_out);
}

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, int renorm,
                        int32_t* idx, float* wts, float* logits_out, cudaStream_t s) {
    return launch_pdl(topk_kernel, dim3((T + 7) / 8), dim3(256), 0, s, logits, bias, T, E, k, renorm, idx,
                      wts, logits_out);
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int cap, int32_t* hist,
                           int32_t* offsets, int32_t* row2ts, int32_t* ts2row, int32_t* meta,
                           int32_t* active, int32_t* tiles, int32_t* pairs, cudaStream_t s, int32_t* zero_words,
                           int n_zero) {
    const int n = T * k;
    const int nblk = (n + kPermChunk - 1) / kPermChunk;
    cudaError_t err = launch_pdl(perm_hist_kernel, dim3(nblk), dim3(256), 0, s, idx, n, E, hist);
    if (err != cudaSuccess) return err;
    return launch_pdl(perm_scatter_kernel, dim3(nblk), dim3(kPermThreads), 0, s, idx, n, E, cap, nblk, hist,
                      offsets, row2ts, ts2row, meta, active, tiles, pairs, zero_words, n_zero);
}

bool route_small_ok(int T, int k) { return (int64_t)T * k <= kRouteSmallMax; }

cudaError_t launch_route_small(const float* logits, const float* bias, int T, int E, int k,
                               int renorm, int cap, int32_t* idx, float* wts, float* logits_out,
                               int32_t* offsets, int32_t* row2ts, int32_t* ts2row, int32_t* meta,
                               int32_t* active, int32_t* tiles, int32_t* pairs, int32_t* zero_words, int n_zero,
                               cudaStream_t s) {
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(route_small_kernel, sizeof(RouteSmallSmem), attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_small_kernel, dim3(1), dim3(kRouteSmallThreads), sizeof(RouteSmallSmem), s, logits,
                      bias, T, E, k, renorm, cap, idx, wts, logits_out, offsets, row2ts, ts2row, meta,
                      active, tiles, pairs, zero_words, n_zero);
}

cudaError_t launch_smooth_quant(const void* x, int in_dtype, const float* inv_s, float act_clip, int T,
                                int d, int k, const int32_t* ts2row, int8_t* xq, float* sx, int8_t* aq,
                                int64_t aq_ld, const float* wts, const int32_t* idx, int fmt, cudaStream_t s) {
    // 256 threads per token with few channel groups each: few registers, so
    // many warps per SM hide the load latency (the kernel is issue- and
    // latency-bound, not bandwidth-bound)
    constexpr int NT = 256;
    const int groups = (d / 8 + NT - 1) / NT;
    auto kern = fmt == FMT_E4M3
                    ? (groups <= 2 ? smooth_quant_kernel<2, FMT_E4M3, NT>
                                   : groups <= 4 ? smooth_quant_kernel<4, FMT_E4M3, NT> : smooth_quant_kernel<8, FMT_E4M3, NT>)
                    : (groups <= 2 ? smooth_quant_kernel<2, FMT_INT8, NT>
                                   : groups <= 4 ? smooth_quant_kernel<4, FMT_INT8, NT> : smooth_quant_kernel<8, FMT_INT8, NT>);
    return launch_pdl(kern, dim3(T), dim3(NT), 0, s, x, in_dtype, inv_s, act_clip, T, d, k, ts2row, xq,
                      sx, aq, aq_ld, wts, idx);
}

cudaError_t launch_ep_read_experts(const uint8_t* recv, int R, int64_t row_bytes, int d, int block_rows,
                                   int ep_first, int n_local, int32_t* idx, int32_t* status, cudaStream_t s) {
    return launch_pdl(ep_read_experts_kernel, dim3((R + 255) / 256), dim3(256), 0, s, recv, R, row_bytes, d,
                      block_rows, ep_first, n_local, idx, status);
}

cudaError_t launch_ep_pack(const uint8_t* send, const int32_t* offsets, const EpRanks& ranks, int world,
                           int block_rows, int64_t row_bytes, uint8_t* blocks, cudaStream_t s) {
    return launch_pdl(ep_pack_kernel, dim3((block_rows + kEpGatherWarps - 1) / kEpGatherWarps, world),
                      dim3(kEpGatherWarps * 32), 0, s, send, offsets, ranks, block_rows, row_bytes, blocks);
}

cudaError_t launch_ep_gather(const uint8_t* recv, int R, int64_t row_bytes, int d, const int32_t* ts2row,
                             int8_t* dst, float* sx, float* wts, cudaStream_t s) {
    return launch_pdl(ep_gather_kernel, dim3((R + kEpGatherWarps - 1) / kEpGatherWarps),
                      dim3(kEpGatherWarps * 32), 0, s, recv, R, row_bytes, d, ts2row, dst, sx, wts);
}

}  // namespace moe
