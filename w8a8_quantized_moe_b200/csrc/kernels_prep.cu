// Offline preparation kernels: SmoothQuant statistics and per-output-channel
// INT8 weight quantisation ("MiniMax-M3 W8A8 on K100AI", s3.2: weights
// per_channel, smooth_quant alpha; s6.1 smoothing moves activation outliers
// into the weights).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Non-negative floats order like their bit patterns, so an integer atomicMax
// on the bits is an exact float max.
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

// absmax[j] = max(absmax[j], max_r |x[r][j]|); grid.x over column blocks of
// 256, grid.y over row slices.
__global__ void calib_absmax_kernel(const void* __restrict__ x, int64_t rows, int d, int dtype,
                                    float* __restrict__ absmax) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= d) return;
    const int64_t per = (rows + gridDim.y - 1) / gridDim.y;
    const int64_t r0 = (int64_t)blockIdx.y * per;
    const int64_t r1 = min(rows, r0 + per);
    float m = 0.0f;
    for (int64_t r = r0; r < r1; ++r) {
        float v = dtype == MOE_BF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(x)[r * d + j])
                                    : reinterpret_cast<const float*>(x)[r * d + j];
        m = fmaxf(m, fabsf(v));
    }
    if (r1 > r0) atomic_max_nonneg(absmax + j, m);
}

// out[r][j] = |fp32(x[r][j] * inv_s[j])|: the smoothed values the per-token
// quantiser sees, for the percentile of the activation clip.
__global__ void scaled_abs_kernel(const void* __restrict__ x, int64_t n, int d, int dtype,
                                  const float* __restrict__ inv_s, float* __restrict__ out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = dtype == MOE_BF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(x)[i])
                                          : reinterpret_cast<const float*>(x)[i];
        out[i] = fabsf(__fmul_rn(v, inv_s[i % d]));
    }
}

// aw[j] = max over experts and output channels of |W_gate[e][j][:]|, |W_up[e][j][:]|
// (one block per (j, e); rows are f contiguous floats).
__global__ void gateup_input_absmax_kernel(const float* __restrict__ wg, const float* __restrict__ wu,
                                           int d, int f, float* __restrict__ aw) {
    __shared__ float red[32];
    const int j = blockIdx.x, e = blockIdx.y;
    const float* g = wg + ((int64_t)e * d + j) * f;
    const float* u = wu + ((int64_t)e * d + j) * f;
    float m = 0.0f;
    for (int n = threadIdx.x; n < f; n += blockDim.x) m = fmaxf(m, fmaxf(fabsf(g[n]), fabsf(u[n])));
    m = block_max_nonneg(m, red);
    if (threadIdx.x == 0) atomic_max_nonneg(aw + j, m);
}

// Per-output-channel quantisation of W [E][K][N] (input j along K, output n
// along N).  Block = (32 channels, expert), 256 threads as 8 rows x 32 columns.
// Pass 1: amax_n = max_j |W'[j][n]| with W' = fp32(s_j * W) (s may be NULL).
// Pass 2: codes rint(W'/sw_n) (INT8) or e4m3(W'/sw_n) (E4M3), sw_n = amax_n /
// 127 or / 448, written K-major to out row map(n).
constexpr int kQCh = 32;
constexpr int kQJ = 128;  // j-chunk staged through shared memory

template <int FMT>
__global__ void __launch_bounds__(256) quantize_channels_kernel(
    const float* __restrict__ w, const float* __restrict__ smooth, int K, int N,
    int8_t* __restrict__ out, int out_rows, int row_block, int row_stride, int row_base,
    float* __restrict__ sw) {
    __shared__ float red[8][kQCh];
    __shared__ float scale_s[kQCh];
    __shared__ __align__(16) int8_t tile[kQCh][kQJ + 16];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int n0 = blockIdx.x * kQCh, e = blockIdx.y;
    const int n = n0 + tx;
    const float* we = w + (int64_t)e * K * N;
    float m = 0.0f;
    if (n < N)
        for (int j = ty; j < K; j += 8) {
            float v = we[(int64_t)j * N + n];
            if (smooth) v = __fmul_rn(smooth[j], v);
            m = fmaxf(m, fabsf(v));
        }
    red[ty][tx] = m;
    __syncthreads();
    if (ty == 0) {
        float a = red[0][tx];
        for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i][tx]);
        const float s = a > 0.0f ? __fdiv_rn(a, fmt_qmax<FMT>()) : 0.0f;
        scale_s[tx] = s;
        if (n < N) sw[(int64_t)e * N + n] = s;
    }
    __syncthreads();
    const float s = scale_s[tx];
    for (int j0 = 0; j0 < K; j0 += kQJ) {
        // codes of channel tx for j0 + ty + 8 i
        for (int i = 0; i < kQJ / 8; ++i) {
            const int jj = ty + 8 * i;
            int q = 0;
            if (n < N && s > 0.0f) {
                float v = we[(int64_t)(j0 + jj) * N + n];
                if (smooth) v = __fmul_rn(smooth[j0 + jj], v);
                q = FMT == FMT_E4M3 ? (int)e4m3_code(__fdiv_rn(v, s)) : quant_code(v, s);
            }
            tile[tx][jj] = (int8_t)q;
        }
        __syncthreads();
        // 32 rows x 128 bytes out, 16 bytes per thread
        const int c = threadIdx.x >> 3, part = threadIdx.x & 7;
        const int nn = n0 + c;
        if (nn < N) {
            const int row = row_base + (nn / row_block) * row_stride + (nn % row_block);
            int8_t* dst = out + ((int64_t)e * out_rows + row) * K + j0 + part * 16;
            *reinterpret_cast<int4*>(dst) = *reinterpret_cast<const int4*>(&tile[c][part * 16]);
        }
        __syncthreads();
    }
}

// Canonical copy of the interleaved gate/up weights: gate[e][n][:], up[e][n][:].
__global__ void export_gateup_kernel(const int8_t* __restrict__ w_gu, int d, int f,
                                     int8_t* __restrict__ gate, int8_t* __restrict__ up) {
    const int n = blockIdx.x, e = blockIdx.y;
    const int base = (n / kGuBlock) * 2 * kGuBlock + (n % kGuBlock);
    const int4* src_g = reinterpret_cast<const int4*>(w_gu + ((int64_t)e * 2 * f + base) * d);
    const int4* src_u = reinterpret_cast<const int4*>(w_gu + ((int64_t)e * 2 * f + base + kGuBlock) * d);
    for (int i = threadIdx.x; i < d / 16; i += blockDim.x) {
        if (gate) reinterpret_cast<int4*>(gate + ((int64_t)e * f + n) * d)[i] = src_g[i];
        if (up) reinterpret_cast<int4*>(up + ((int64_t)e * f + n) * d)[i] = src_u[i];
    }
}

}  // namespace

cudaError_t launch_calib_absmax(const void* x, int64_t rows, int d, int dtype, float* absmax,
                                cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    dim3 grid((d + 255) / 256, (unsigned)(rows < 64 ? rows : 64));
    calib_absmax_kernel<<<grid, 256, 0, s>>>(x, rows, d, dtype, absmax);
    return cudaGetLastError();
}

cudaError_t launch_scaled_abs(const void* x, int64_t rows, int d, int dtype, const float* inv_s, float* out,
                              cudaStream_t s) {
    const int64_t n = rows * d;
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = (n + 255) / 256;
    scaled_abs_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(x, n, d, dtype, inv_s, out);
    return cudaGetLastError();
}

cudaError_t launch_gateup_input_absmax(const float* w_gate, const float* w_up, int E, int d, int f,
                                       float* aw, cudaStream_t s) {
    gateup_input_absmax_kernel<<<dim3(d, E), 256, 0, s>>>(w_gate, w_up, d, f, aw);
    return cudaGetLastError();
}

cudaError_t launch_quantize_channels(const float* w, const float* smooth, int E, int K, int N,
                                     int8_t* out, int out_rows, int row_block, int row_stride,
                                     int row_base, float* sw, int fmt, cudaStream_t s) {
    dim3 grid((N + kQCh - 1) / kQCh, E);
    if (fmt == FMT_E4M3)
        quantize_channels_kernel<FMT_E4M3><<<grid, 256, 0, s>>>(w, smooth, K, N, out, out_rows, row_block,
                                                                row_stride, row_base, sw);
    else
        quantize_channels_kernel<FMT_INT8><<<grid, 256, 0, s>>>(w, smooth, K, N, out, out_rows, row_block,
                                                                row_stride, row_base, sw);
    return cudaGetLastError();
}

cudaError_t launch_export_gateup(const int8_t* w_gu, int E, int d, int f, int8_t* gate, int8_t* up,
                                 cudaStream_t s) {
    export_gateup_kernel<<<dim3(f, E), 128, 0, s>>>(w_gu, d, f, gate, up);
    return cudaGetLastError();
}

}  // namespace moe
