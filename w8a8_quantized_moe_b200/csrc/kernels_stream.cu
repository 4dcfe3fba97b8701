// Weight-streaming expert path for small token counts (decode).
//
// With few rows per expert the layer is bound by reading the active experts'
// INT8 weights ("MiniMax-M3 W8A8 on K100AI", s1.1-1.3: decode is weight-
// bandwidth bound and INT8 halves the bytes).  Each active expert's weight
// rows are streamed once with 128-bit loads that bypass L1; a warp owns a
// few output channels and splits K across its lanes (16 bytes per lane per
// 512-byte segment), accumulating INT8 x INT8 products with dp4a and
// reducing across lanes with shuffles.  Integer sums are exact, so the
// accumulators equal the grouped-GEMM definition bit for bit.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kStThreads = 256;
constexpr int kStWarps = kStThreads / 32;
constexpr int kStRows = 8;       // rows of one expert processed per pass over its weights
constexpr int kStSegMax = 16;    // 512-byte K segments held in flight per channel per pass
constexpr int kStMaxK = 16384;   // largest d and f a layer may have: the staged rows take kStRows x K bytes

// acc[r][c] = sum_k A[r][k] * W[ch_c][k] for the nr rows staged in smem (row
// stride K) and CH consecutive weight rows starting at wrow (stride K).
template <int CH>
__device__ __forceinline__ void stream_dot(const int8_t* __restrict__ wrow, int K,
                                           const int8_t* __restrict__ As, int nr, int lane,
                                           int acc[kStRows][CH]) {
#pragma unroll
    for (int r = 0; r < kStRows; ++r)
#pragma unroll
        for (int c = 0; c < CH; ++c) acc[r][c] = 0;
    const int nseg = (K + 511) / 512;
    for (int s0 = 0; s0 < nseg; s0 += kStSegMax / CH) {
        int4 wv[kStSegMax / CH][CH];
#pragma unroll
        for (int si = 0; si < kStSegMax / CH; ++si) {
            const int off = (s0 + si) * 512 + lane * 16;
#pragma unroll
            for (int c = 0; c < CH; ++c)
                wv[si][c] = (s0 + si < nseg && off < K) ? ld_stream_v4(wrow + (int64_t)c * K + off)
                                                        : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int si = 0; si < kStSegMax / CH; ++si) {
            const int off = (s0 + si) * 512 + lane * 16;
            if (s0 + si >= nseg || off >= K) continue;
#pragma unroll
            for (int r = 0; r < kStRows; ++r) {
                if (r >= nr) break;
                const int4 a = *reinterpret_cast<const int4*>(As + r * K + off);
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    int v = acc[r][c];
                    v = dp4a(wv[si][c].x, a.x, v);
                    v = dp4a(wv[si][c].y, a.y, v);
                    v = dp4a(wv[si][c].z, a.z, v);
                    v = dp4a(wv[si][c].w, a.w, v);
                    acc[r][c] = v;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kStRows; ++r) {
        if (r >= nr) break;
#pragma unroll
        for (int c = 0; c < CH; ++c) acc[r][c] = warp_sum_i(acc[r][c]);
    }
}

// Gate/up: unit = (active expert, block of 8*CH*... channels).  Writes acc1 in
// canonical channel order (gate 0..f-1 | up 0..f-1).
constexpr int kGuCh = 2;                              // channels per warp step
constexpr int kGuUnit = kStWarps * kGuCh * 4;         // 64 channels per unit

__global__ void __launch_bounds__(kStThreads) stream_gateup_kernel(
    const int8_t* __restrict__ w_gu, int d, int f, int k, const int8_t* __restrict__ xq,
    const int32_t* __restrict__ row2ts, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ active, const int32_t* __restrict__ meta,
    int32_t* __restrict__ acc1) {    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) int8_t As[];   // [kStRows][d]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_units_e = (2 * f) / kGuUnit;
    const int total = meta[META_NACTIVE] * n_units_e;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int e = active[u / n_units_e];
        const int ch0 = (u % n_units_e) * kGuUnit;
        const int r0 = offsets[e], cnt = offsets[e + 1] - r0;
        for (int c0 = 0; c0 < cnt; c0 += kStRows) {
            const int nr = min(kStRows, cnt - c0);
            __syncthreads();
            for (int i = threadIdx.x; i < nr * (d / 16); i += blockDim.x) {
                const int r = i / (d / 16), part = i % (d / 16);
                const int t = row2ts[r0 + c0 + r] / k;
                reinterpret_cast<int4*>(As + r * d)[part] =
                    reinterpret_cast<const int4*>(xq + (int64_t)t * d)[part];
            }
            __syncthreads();
            for (int step = 0; step < kGuUnit / (kStWarps * kGuCh); ++step) {
                const int ch = ch0 + (step * kStWarps + warp) * kGuCh;   // interleaved channel
                int acc[kStRows][kGuCh];
                stream_dot<kGuCh>(w_gu + ((int64_t)e * 2 * f + ch) * d, d, As, nr, lane, acc);
#pragma unroll
                for (int r = 0; r < kStRows; ++r) {
                    if (r >= nr) break;
#pragma unroll
                    for (int c = 0; c < kGuCh; ++c) {
                        if (lane != r * kGuCh + c) continue;
                        const int chi = ch + c;
                        const int blk = chi / (2 * kGuBlock), within = chi % (2 * kGuBlock);
                        const int is_up = within >= kGuBlock;
                        const int n = blk * kGuBlock + (within % kGuBlock);
                        acc1[(int64_t)(r0 + c0 + r) * 2 * f + is_up * f + n] = acc[r][c];
                    }
                }
            }
        }
    }
}

// SwiGLU + per-row requantisation of h ("MiniMax-M3 W8A8 on K100AI", s4.3:
// the expert intermediate stays INT8 between the two matmuls).  One block per
// row: g = fp32(fp32(acc_g sx) sw_g), u likewise, h = silu(g) u, then the INT8
// rule over the f values of the row.
constexpr int kSwThreads = 256;

__global__ void __launch_bounds__(kSwThreads) swiglu_requant_kernel(
    const int32_t* __restrict__ acc1, int f, int k, const int32_t* __restrict__ row2ts,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ sx,
    const float* __restrict__ sw_gate, const float* __restrict__ sw_up,
    const int32_t* __restrict__ meta, int8_t* __restrict__ hq, float* __restrict__ sh) {    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) float hs[];   // [f]
    __shared__ float red[32];
    const int r = blockIdx.x;
    if (r >= meta[META_R]) return;
    const int ts = row2ts[r];
    const int e = topk_idx[ts];
    const float sxt = sx[ts / k];
    const int32_t* ag = acc1 + (int64_t)r * 2 * f;
    const int32_t* au = ag + f;
    const float* swg = sw_gate + (int64_t)e * f;
    const float* swu = sw_up + (int64_t)e * f;
    float m = 0.0f;
    for (int g4 = threadIdx.x; g4 < f / 4; g4 += blockDim.x) {
        const int4 a = reinterpret_cast<const int4*>(ag)[g4];
        const int4 b = reinterpret_cast<const int4*>(au)[g4];
        const float4 s1 = reinterpret_cast<const float4*>(swg)[g4];
        const float4 s2 = reinterpret_cast<const float4*>(swu)[g4];
        const int av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
        const float gs[4] = {s1.x, s1.y, s1.z, s1.w}, us[4] = {s2.x, s2.y, s2.z, s2.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float g = __fmul_rn(__fmul_rn(__int2float_rn(av[c]), sxt), gs[c]);
            const float u = __fmul_rn(__fmul_rn(__int2float_rn(bv[c]), sxt), us[c]);
            const float h = __fmul_rn(moe_silu(g), u);
            hs[g4 * 4 + c] = h;
            m = fmaxf(m, fabsf(h));
        }
    }
    const float amax = block_max_nonneg(m, red);   // includes a __syncthreads for hs
    const float s = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    if (threadIdx.x == 0) sh[r] = s;
    for (int g4 = threadIdx.x; g4 < f / 4; g4 += blockDim.x) {
        const float4 h = reinterpret_cast<const float4*>(hs)[g4];
        const uint32_t p = s > 0.0f ? pack4(quant_code(h.x, s), quant_code(h.y, s),
                                            quant_code(h.z, s), quant_code(h.w, s))
                                    : 0u;
        reinterpret_cast<uint32_t*>(hq + (int64_t)r * f)[g4] = p;
    }
}

// Down projection: unit = (active expert, 128 output channels); rows of the
// expert are contiguous in hq.  Epilogue o = fp32(fp32(fp32(acc2 sh) sw) w).
constexpr int kDnCh = 4;
constexpr int kDnUnit = kStWarps * kDnCh * 4;   // 128 channels per unit

__global__ void __launch_bounds__(kStThreads) stream_down_kernel(
    const int8_t* __restrict__ w_dn, int d, int f, const int8_t* __restrict__ hq,
    const float* __restrict__ sh, const int32_t* __restrict__ row2ts,
    const float* __restrict__ topk_w, const float* __restrict__ sw_dn,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ active,
    const int32_t* __restrict__ meta, void* __restrict__ o, int o_bf16, int32_t* __restrict__ acc2_dbg) {    pdl_wait();
    pdl_trigger();

    extern __shared__ __align__(16) int8_t As[];   // [kStRows][f]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_units_e = d / kDnUnit;
    const int total = meta[META_NACTIVE] * n_units_e;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int e = active[u / n_units_e];
        const int ch0 = (u % n_units_e) * kDnUnit;
        const int r0 = offsets[e], cnt = offsets[e + 1] - r0;
        for (int c0 = 0; c0 < cnt; c0 += kStRows) {
            const int nr = min(kStRows, cnt - c0);
            __syncthreads();
            for (int i = threadIdx.x; i < nr * (f / 16); i += blockDim.x)
                reinterpret_cast<int4*>(As)[i] =
                    reinterpret_cast<const int4*>(hq + (int64_t)(r0 + c0) * f)[i];
            __syncthreads();
            for (int step = 0; step < kDnUnit / (kStWarps * kDnCh); ++step) {
                const int ch = ch0 + (step * kStWarps + warp) * kDnCh;
                int acc[kStRows][kDnCh];
                stream_dot<kDnCh>(w_dn + ((int64_t)e * d + ch) * f, f, As, nr, lane, acc);
#pragma unroll
                for (int r = 0; r < kStRows; ++r) {
                    if (r >= nr) break;
#pragma unroll
                    for (int c = 0; c < kDnCh; ++c) {
                        if (lane != r * kDnCh + c) continue;
                        const int row = r0 + c0 + r;
                        const int n = ch + c;
                        const float v = __fmul_rn(__fmul_rn(__fmul_rn(__int2float_rn(acc[r][c]), sh[row]),
                                                            sw_dn[(int64_t)e * d + n]),
                                                  topk_w[row2ts[row]]);
                        if (o_bf16)
                            reinterpret_cast<uint16_t*>(o)[(int64_t)row * d + n] = f32_to_bf16_bits(v);
                        else
                            reinterpret_cast<float*>(o)[(int64_t)row * d + n] = v;
                        if (acc2_dbg) acc2_dbg[(int64_t)row * d + n] = acc[r][c];
                    }
                }
            }
        }
    }
}

// Un-sort + weighted sum: y[t] = ((0 + o_slot0) + o_slot1) + ... over the kept
// slots, in slot order, then cast to the output dtype.  O16: the per-slot rows
// are bf16 (bf16-output layers), else fp32.  A thread owns 8 channels of one
// token: the token's row indices first, then all kept slots' loads (16 bytes
// each for bf16 rows) in flight together, then the sum in slot order.
// Where a sorted row's output sits in fixed blocks returned by the ranks of
// an expert-parallel exchange: row r of rank g's experts (rows
// [offsets[first[g]], offsets[first[g + 1]])) is row 1 + r - offsets[first[g]]
// of block g (blocks of block_rows rows; row 0 is the header).
struct BlockMap {
    const int32_t* offsets;   // null: rows are not blocked
    EpRanks ranks;
    int world, block_rows;
};

__device__ __forceinline__ int block_row(const BlockMap& bm, int r) {
    int g = 0;
    while (g + 1 < bm.world && r >= bm.offsets[bm.ranks.first[g + 1]]) ++g;
    return g * bm.block_rows + 1 + r - bm.offsets[bm.ranks.first[g]];
}

// KM: the largest k the instance serves (4 or kMaxK): the slot arrays live in
// registers, so a smaller bound leaves room for more warps per SM.
template <bool O16, bool BLOCKED, int KM>
__global__ void combine_kernel(const void* __restrict__ o, const int32_t* __restrict__ ts2row,
                               int k, int d, int out_dtype, void* __restrict__ y, const BlockMap bm) {
    pdl_wait();
    pdl_trigger();

    const int t = blockIdx.x;
    const int n8 = blockIdx.y * blockDim.x + threadIdx.x;
    if (n8 * 8 >= d) return;
    int rows[KM];
#pragma unroll
    for (int s = 0; s < KM; ++s) rows[s] = s < k ? ts2row[(int64_t)t * k + s] : -1;
    if (BLOCKED) {
#pragma unroll
        for (int s = 0; s < KM; ++s)
            if (rows[s] >= 0) rows[s] = block_row(bm, rows[s]);
    }
    // loads of every kept slot first (raw 16-byte words: few registers, so many
    // warps per SM), then the sum in slot order
    uint4 raw[KM][O16 ? 1 : 2];
#pragma unroll
    for (int s = 0; s < KM; ++s) {
        if (rows[s] < 0) continue;
        if (O16) {
            raw[s][0] = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(o) + (int64_t)rows[s] * d)[n8];
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(o) + (int64_t)rows[s] * d);
            raw[s][0] = src[2 * n8];
            raw[s][O16 ? 0 : 1] = src[2 * n8 + 1];
        }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < KM; ++s) {
        if (rows[s] < 0) continue;
        float v[8];
        if (O16) {
            const uint32_t w[4] = {raw[s][0].x, raw[s][0].y, raw[s][0].z, raw[s][0].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
        } else {
            const uint32_t w[8] = {raw[s][0].x, raw[s][0].y, raw[s][0].z, raw[s][0].w,
                                   raw[s][O16 ? 0 : 1].x, raw[s][O16 ? 0 : 1].y, raw[s][O16 ? 0 : 1].z,
                                   raw[s][O16 ? 0 : 1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(w[i]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = __fadd_rn(acc[c], v[c]);
    }
    if (out_dtype == MOE_BF16) {
        uint32_t p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            p[i] = (uint32_t)f32_to_bf16_bits(acc[2 * i]) | ((uint32_t)f32_to_bf16_bits(acc[2 * i + 1]) << 16);
        reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + (int64_t)t * d)[n8] = make_uint4(p[0], p[1], p[2], p[3]);
    } else {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + (int64_t)t * d);
        dst[2 * n8] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[2 * n8 + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

int stream_grid(const moe_w8a8_weights* w, int units_upper) {
    return max(1, min(units_upper, w->num_sms * 2));
}

}  // namespace

cudaError_t launch_stream_gateup(const moe_w8a8_weights* w, int T, const int8_t* xq,
                                 const int32_t* row2ts, const int32_t* offsets,
                                 const int32_t* active, const int32_t* meta, int32_t* acc1,
                                 cudaStream_t s) {
    const int d = w->cfg.d, f = w->cfg.f;
    const size_t smem = (size_t)kStRows * d;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(stream_gateup_kernel, (size_t)kStRows * kStMaxK, attr);
    if (e != cudaSuccess) return e;
    const int grid = stream_grid(w, w->cfg.n_experts * (2 * f / kGuUnit));
    (void)T;
    return launch_pdl(stream_gateup_kernel, dim3(grid), dim3(kStThreads), smem, s, w->w_gu, d, f,
                      w->cfg.top_k, xq, row2ts, offsets, active, meta, acc1);
}

cudaError_t launch_swiglu_requant(const moe_w8a8_weights* w, const int32_t* acc1,
                                  const int32_t* row2ts, const int32_t* topk_idx, const float* sx,
                                  const int32_t* meta, int max_rows, int8_t* hq, float* sh,
                                  cudaStream_t s) {
    const int f = w->cfg.f;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(swiglu_requant_kernel, 100 * 1024, attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(swiglu_requant_kernel, dim3(max_rows), dim3(kSwThreads), (size_t)f * 4, s, acc1, f,
                      w->cfg.top_k, row2ts, topk_idx, sx, w->sw_gate, w->sw_up, meta, hq, sh);
}

cudaError_t launch_stream_down(const moe_w8a8_weights* w, int T, const int8_t* hq, const float* sh,
                               const int32_t* row2ts, const float* topk_w, const int32_t* offsets,
                               const int32_t* active, const int32_t* meta, void* o,
                               int32_t* acc2_dbg, cudaStream_t s) {
    const int d = w->cfg.d, f = w->cfg.f;
    const size_t smem = (size_t)kStRows * f;
    const int grid = stream_grid(w, w->cfg.n_experts * (d / kDnUnit));
    (void)T;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(stream_down_kernel, (size_t)kStRows * kStMaxK, attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(stream_down_kernel, dim3(grid), dim3(kStThreads), smem, s, w->w_dn, d, f, hq, sh,
                      row2ts, topk_w, w->sw_dn, offsets, active, meta, o, (int)(w->cfg.out_dtype == MOE_BF16),
                      acc2_dbg);
}

cudaError_t launch_combine(const void* o, int o_bf16, const int32_t* ts2row, int T, int k, int d,
                           int out_dtype, void* y, cudaStream_t s) {
    dim3 grid(T, (d / 8 + 255) / 256);
    const BlockMap none{};
    auto kern = o_bf16 ? (k <= 4 ? combine_kernel<true, false, 4> : combine_kernel<true, false, kMaxK>)
                       : (k <= 4 ? combine_kernel<false, false, 4> : combine_kernel<false, false, kMaxK>);
    return launch_pdl(kern, grid, dim3(256), 0, s, o, ts2row, k, d, out_dtype, y, none);
}

cudaError_t launch_combine_blocked(const float* o_blocks, const int32_t* ts2row, const int32_t* offsets,
                                   const EpRanks& ranks, int world, int block_rows, int T, int k, int d,
                                   int out_dtype, void* y, cudaStream_t s) {
    dim3 grid(T, (d / 8 + 255) / 256);
    const BlockMap bm{offsets, ranks, world, block_rows};
    auto kern = k <= 4 ? combine_kernel<false, true, 4> : combine_kernel<false, true, kMaxK>;
    return launch_pdl(kern, grid, dim3(256), 0, s, (const void*)o_blocks, ts2row, k, d, out_dtype, y, bm);
}

}  // namespace moe
