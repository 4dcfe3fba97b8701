// Device-side helpers shared by the kernels of the W8A8 MoE layer.
//
// Every floating-point step that decides an integer (a quantised code, a
// top-k choice) is written with explicit round-to-nearest intrinsics so that
// the compiler cannot contract or reorder it: the layer's specification fixes
// each of those operations as one IEEE fp32 operation in a stated order.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace moe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// exp by Cody & Waite range reduction and a degree-7 Taylor polynomial.
// x is clamped to [-87, 88]; x = n ln2 + r with n = rint(x log2 e); ln2 is
// split into a head with 16 significant bits (n * head exact for |n| < 256)
// and an fp32 tail; e^r = sum_{i<=7} r^i / i! in Horner form (|r| <= ln2/2);
// 2^n is assembled from exponent bits (n in [-126, 127], always normal).
// This fixed sequence is what makes SiLU and the gate softmax reproducible
// bit for bit against a CPU evaluation of the same steps.
// ---------------------------------------------------------------------------
namespace expc {
constexpr double kLn2 = 0.69314718055994530941723212145818;
constexpr double fact(int i) { return i <= 1 ? 1.0 : i * fact(i - 1); }
constexpr float kLog2e = (float)(1.0 / kLn2);
constexpr float kLn2Hi = (float)((double)(long long)(kLn2 * 65536.0) / 65536.0);
constexpr float kLn2Lo = (float)(kLn2 - (double)kLn2Hi);
constexpr float kC0 = (float)(1.0 / fact(0)), kC1 = (float)(1.0 / fact(1));
constexpr float kC2 = (float)(1.0 / fact(2)), kC3 = (float)(1.0 / fact(3));
constexpr float kC4 = (float)(1.0 / fact(4)), kC5 = (float)(1.0 / fact(5));
constexpr float kC6 = (float)(1.0 / fact(6)), kC7 = (float)(1.0 / fact(7));
}  // namespace expc

__device__ __forceinline__ float moe_exp(float x) {
    using namespace expc;
    x = fminf(fmaxf(x, -87.0f), 88.0f);
    const float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = kC7;
    p = __fmaf_rn(p, r, kC6);
    p = __fmaf_rn(p, r, kC5);
    p = __fmaf_rn(p, r, kC4);
    p = __fmaf_rn(p, r, kC3);
    p = __fmaf_rn(p, r, kC2);
    p = __fmaf_rn(p, r, kC1);
    p = __fmaf_rn(p, r, kC0);
    const int ni = __float2int_rn(n);
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

// silu(g) = g / (1 + e^-g)
__device__ __forceinline__ float moe_silu(float g) {
    return __fdiv_rn(g, __fadd_rn(1.0f, moe_exp(-g)));
}

// Symmetric INT8 code of v for scale s > 0: rint(v / s), ties to even, clamped
// to [-127, 127].  Callers handle s == 0 (all-zero vector -> code 0).
__device__ __forceinline__ int quant_code(float v, float s) {
    int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

// The same code without a division in the common case.  With r = fp32(1/s)
// and t = fp32(v r), |t - fp32(v / s)| <= 3.0001 u |v / s| (u = 2^-24) by the
// standard rounding-error bound, i.e. below 2.3e-5 for |v / s| <= 128.  So
// unless t lies within 3e-5 of a half-integer, t and the IEEE quotient round
// to the same integer; near a half-integer the IEEE quotient is formed.  The
// result is identical to quant_code(v, s).  `r` must be fp32(1 / s), s > 0;
// when 1/s overflows (s below 2^-128, a row whose largest value is under
// about 3.7e-37) the bound does not hold and the quotient is formed.
__device__ __forceinline__ int quant_code_fast(float v, float s, float r) {
    if (isinf(r)) return quant_code(v, s);
    const float t = __fmul_rn(v, r);
    const float n = rintf(t);
    const float dist = fabsf(fabsf(__fsub_rn(t, n)) - 0.5f);
    int q = (dist > 3.0e-5f || fabsf(t) > 130.0f) ? __float2int_rn(n) : __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

// E4M3 code of v: the nearest E4M3 value, ties to even, magnitudes beyond 448
// saturated (the conversion instruction's round-to-nearest, satfinite mode).
__device__ __forceinline__ uint32_t e4m3_code(float v) {
    return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Expert number formats (values of moe_w8a8_config::expert_format).
enum { FMT_INT8 = 0, FMT_E4M3 = 1 };

// Largest code magnitude of a format: the scale of a vector is amax / this.
template <int FMT>
__device__ __forceinline__ float fmt_qmax() { return FMT == FMT_E4M3 ? 448.0f : 127.0f; }

// Code byte of v for scale s > 0 (r = fp32(1 / s), used by the INT8 rule only).
template <int FMT>
__device__ __forceinline__ uint32_t fmt_code(float v, float s, float r) {
    if (FMT == FMT_E4M3) return e4m3_code(__fdiv_rn(v, s));
    return (uint32_t)quant_code_fast(v, s, r) & 0xffu;
}

// Pack four INT8 codes (low byte first).
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// The four code bytes of v0..v3 for scale s > 0 (r = fp32(1 / s)), packed low
// byte first: identical to fmt_code element by element.  For INT8 the four
// products t = v r are rounded together and the near-half-integer test of
// quant_code_fast is combined into one branch: if any element needs the IEEE
// quotient (or 1/s overflowed), all four are formed by quant_code, which gives
// the same codes for the others (the test's premise).
template <int FMT>
__device__ __forceinline__ uint32_t fmt_codes4(float v0, float v1, float v2, float v3, float s, float r) {
    if (FMT == FMT_E4M3)
        return pack4((int)fmt_code<FMT>(v0, s, r), (int)fmt_code<FMT>(v1, s, r), (int)fmt_code<FMT>(v2, s, r),
                     (int)fmt_code<FMT>(v3, s, r));
    const float v[4] = {v0, v1, v2, v3};
    float n[4];
    bool slow = isinf(r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float t = __fmul_rn(v[i], r);
        n[i] = rintf(t);
        const float dist = fabsf(fabsf(__fsub_rn(t, n[i])) - 0.5f);
        slow |= dist <= 3.0e-5f && fabsf(t) <= 130.0f;
    }
    int q[4];
    if (!slow) {
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = max(-127, min(127, __float2int_rn(n[i])));
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = quant_code(v[i], s);
    }
    return pack4(q[0], q[1], q[2], q[3]);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float((uint32_t)h << 16);
}

// fp32 -> bf16 round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Streaming 128-bit global load that does not allocate in L1 (weights are
// read once per launch).
__device__ __forceinline__ int4 ld_stream_v4(const void* p) {
    int4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ int dp4a(int a, int b, int c) { return __dp4a(a, b, c); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Max of non-negative floats over a block (blockDim.x multiple of 32, <= 1024).
// Exact: max does not depend on the order.  `red` needs 32 floats.
__device__ __forceinline__ float block_max_nonneg(float v, float* red) {
    v = warp_max(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    const int nw = blockDim.x >> 5;
    float m = lane < nw ? red[lane] : 0.0f;
    m = warp_max(m);
    return m;
}

// Load 8 consecutive activations as fp32 (in_dtype: 0 fp32, 1 bf16).
__device__ __forceinline__ void load8_act(const void* x, int64_t idx, int in_dtype, float v[8]) {
    if (in_dtype == 1) {
        const int4 raw = *reinterpret_cast<const int4*>(reinterpret_cast<const uint16_t*>(x) + idx);
        const uint32_t w[4] = {(uint32_t)raw.x, (uint32_t)raw.y, (uint32_t)raw.z, (uint32_t)raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + idx);
        const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + idx + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// Programmatic dependent launch: every kernel of a forward lets the next one be
// scheduled as soon as it starts (trigger) and waits for the previous kernel's
// results before touching any shared buffer (wait).  Both are no-ops for a
// kernel launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace moe

// Host: raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per device (function attributes belong to each device's
// context; `done` holds one bit per device that has it).
template <typename... KArgs>
inline cudaError_t smem_attr_once(void (*kernel)(KArgs...), size_t bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Host: launch `kernel` on `s` with programmatic stream serialization allowed,
// so that it may start while the previous kernel on the stream finishes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
