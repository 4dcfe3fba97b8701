/*
 * Seeded synthetic inputs for the W8A8 MoE layer.
 *
 * This module only draws numbers: it holds none of the layer's arithmetic
 * (no smoothing, quantisation, routing, GEMM or combine).  Both the CPU
 * oracle and the CUDA path are fed from the arrays it writes, so the two
 * sides always see identical bytes.
 *
 * Generator: every value is a pure function of (seed, tensor id, element
 * index).  The bits come from the SplitMix64 sequence (Steele, Lea and
 * Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):
 * state_i = base + (i + 1) * 0x9E3779B97F4A7C15, output = mix64(state_i)
 * with the mix64 finaliser of that paper.  Because element i depends on i
 * alone, any slice can be produced independently and in parallel.
 *
 * Uniforms take the top 53 bits: u = (r >> 11) * 2^-53, in [0, 1).
 * Normals use the Box-Muller transform in fp64 on the pair (2j, 2j+1):
 * rho = sqrt(-2 ln(1 - u_2j)), z_2j = rho cos(2 pi u_2j+1),
 * z_2j+1 = rho sin(2 pi u_2j+1), then mean + std * z rounded once to fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream base for one tensor: the seed and the tensor id are mixed so that
 * neighbouring seeds or ids give unrelated streams. */
static inline uint64_t stream_base(uint64_t seed, uint32_t tensor_id) {
    return mix64(mix64(seed + GOLDEN) ^ ((uint64_t)tensor_id * 0xD1B54A32D192ED03ULL));
}

static inline uint64_t draw_bits(uint64_t base, uint64_t i) {
    return mix64(base + (i + 1) * GOLDEN);
}

static inline double draw_uniform(uint64_t base, uint64_t i) {
    return (double)(draw_bits(base, i) >> 11) * (1.0 / 9007199254740992.0);
}

static inline double draw_normal(uint64_t base, uint64_t i) {
    uint64_t j = i >> 1;
    double u1 = draw_uniform(base, 2 * j);
    double u2 = draw_uniform(base, 2 * j + 1);
    double rho = sqrt(-2.0 * log(1.0 - u1));
    double ang = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? rho * sin(ang) : rho * cos(ang);
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
static inline uint16_t f32_to_bf16_bits(float v) {
    uint32_t b;
    memcpy(&b, &v, 4);
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

static inline float bf16_bits_to_f32(uint16_t h) {
    uint32_t b = (uint32_t)h << 16;
    float v;
    memcpy(&v, &b, 4);
    return v;
}

/* out[i] = fp32(mean + std * z_{start+i}), z ~ N(0,1). */
void synth_normal_f32(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t n,
                      double mean, double std, float* out) {
    uint64_t base = stream_base(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = (float)(mean + std * draw_normal(base, start + (uint64_t)i));
}

/* out[i] = fp32(lo + (hi - lo) * u_{start+i}), u ~ U[0,1). */
void synth_uniform_f32(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t n,
                       double lo, double hi, float* out) {
    uint64_t base = stream_base(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = (float)(lo + (hi - lo) * draw_uniform(base, start + (uint64_t)i));
}

/* Raw 64-bit draws (used to build permutations and channel subsets). */
void synth_bits_u64(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t n, uint64_t* out) {
    uint64_t base = stream_base(seed, tensor_id);
    for (uint64_t i = 0; i < n; ++i) out[i] = draw_bits(base, start + i);
}

typedef struct { uint64_t key; int32_t idx; } keyed_t;

static int cmp_keyed(const void* a, const void* b) {
    const keyed_t* x = (const keyed_t*)a;
    const keyed_t* y = (const keyed_t*)b;
    if (x->key != y->key) return x->key < y->key ? -1 : 1;
    return x->idx < y->idx ? -1 : (x->idx > y->idx);
}

/* A seeded permutation of 0..n-1: sort indices by their random keys
 * (ties, which are practically impossible, go to the lower index). */
void synth_permutation(uint64_t seed, uint32_t tensor_id, int32_t n, int32_t* out) {
    keyed_t* kv = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)(n > 0 ? n : 1));
    uint64_t base = stream_base(seed, tensor_id);
    for (int32_t i = 0; i < n; ++i) { kv[i].key = draw_bits(base, (uint64_t)i); kv[i].idx = i; }
    qsort(kv, (size_t)n, sizeof(keyed_t), cmp_keyed);
    for (int32_t i = 0; i < n; ++i) out[i] = kv[i].idx;
    free(kv);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* A seeded subset of m channels out of d, returned in ascending order:
 * the first m entries of a seeded permutation. */
void synth_subset(uint64_t seed, uint32_t tensor_id, int32_t d, int32_t m, int32_t* out) {
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(d > 0 ? d : 1));
    synth_permutation(seed, tensor_id, d, perm);
    for (int32_t i = 0; i < m; ++i) out[i] = perm[i];
    qsort(out, (size_t)m, sizeof(int32_t), cmp_i32);
    free(perm);
}

/*
 * Token activations X [rows][d]: N(0,1) per element, with the listed outlier
 * channels multiplied by `factor` before rounding.  Rows are numbered from
 * `row0` so that a slice of a big draw can be made on its own.  With
 * as_bf16 != 0 the fp32 value is rounded to bf16 (nearest even); both the
 * bf16 bits (out_bits, may be NULL) and their exact fp32 value (out_f32, may
 * be NULL) are written.
 */
void synth_activations(uint64_t seed, uint32_t tensor_id, int64_t row0, int64_t rows, int32_t d,
                       const int32_t* outlier_channels, int32_t n_outliers, double factor,
                       int32_t as_bf16, float* out_f32, uint16_t* out_bits) {
    uint64_t base = stream_base(seed, tensor_id);
    double* mult = (double*)malloc(sizeof(double) * (size_t)d);
    for (int32_t j = 0; j < d; ++j) mult[j] = 1.0;
    for (int32_t i = 0; i < n_outliers; ++i) mult[outlier_channels[i]] = factor;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t j = 0; j < d; ++j) {
            uint64_t gi = (uint64_t)(row0 + r) * (uint64_t)d + (uint64_t)j;
            float v = (float)(mult[j] * draw_normal(base, gi));
            if (as_bf16) {
                uint16_t h = f32_to_bf16_bits(v);
                if (out_bits) out_bits[r * d + j] = h;
                v = bf16_bits_to_f32(h);
            }
            if (out_f32) out_f32[r * d + j] = v;
        }
    }
    free(mult);
}

/* fp32 -> bf16 bits (nearest even), for callers that build bf16 tensors. */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_bits(in[i]);
}
