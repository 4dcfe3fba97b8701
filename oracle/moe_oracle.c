/*
 * CPU oracle of the W8A8 mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * library: both follow the same written specification independently.
 *
 * Plain single-threaded C, compiled with -ffp-contract=off so that every
 * fp32 operation is one IEEE round-to-nearest-even operation in the order
 * written here (fmaf only where a fused multiply-add is written).
 *
 * Sources (page title, section):
 *  [MiniMax-M3 W8A8 on K100AI] mhpq.cn "MetaInfer ... MiniMax-M3 W8A8" page:
 *     s1.2 (W8A8: INT8 weights x INT8 activations on the INT8 GEMM path,
 *     accumulate, dequantise), s3.2 (per-channel weights, per-token
 *     activations, SmoothQuant alpha = 0.6), s4.3 (stay in the INT8 domain
 *     between the expert matmuls; fuse the expert FFN), s6.4 (per-token
 *     quantisation and smoothing as the first two defences against outliers).
 *  [Day0 adaptation] ruibaoantu.com "Day0 adaptation of ultra-large model
 *     inference" page, section 4 "MoE operator fusion": gate, sort,
 *     grouped GEMM, un-sort and weighted sum; top-k routing must match the
 *     reference exactly including the tie-break rule.  Section 2 item 2:
 *     expert capacity factor, overflow tokens dropped.
 * The pages give no formulas beyond these; every fixed order or rounding
 * below is a reading, marked READING, and is the specification both sides
 * implement.
 *
 * Pins (what checks this file against something other than itself) live in
 * tests/test_oracle_*.py.  Functions whose exact rounding is fixed only by a
 * READING (router partial-sum order, the exp polynomial) are pinned by
 * bounds, brute force and closed forms, not by the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* exp: Cody & Waite range reduction + Taylor polynomial (READING: the pages */
/* fix no exp; a written-out exp makes SiLU and the gate softmax, and hence  */
/* the INT8 h codes, reproducible bit for bit on both sides).                */
/* ------------------------------------------------------------------------ */

/* x = n ln2 + r with n = rint(x / ln2); ln2 split into a 16-significant-bit
 * head (so n * head is exact for |n| < 256) and an fp32 tail; e^r by its
 * Taylor series to degree 7 (|r| <= ln2/2, truncation < 0.05 ulp); the
 * result scaled by 2^n built from exponent bits. */
static float EXP_LOG2E, EXP_LN2_HI, EXP_LN2_LO, EXP_C[8];
static int exp_ready = 0;

static void exp_init(void) {
    const double ln2 = 0.69314718055994530941723212145818;
    EXP_LOG2E = (float)(1.0 / ln2);
    EXP_LN2_HI = (float)(floor(ln2 * 65536.0) / 65536.0);
    EXP_LN2_LO = (float)(ln2 - (double)EXP_LN2_HI);
    double fact = 1.0;
    for (int i = 0; i < 8; ++i) {
        if (i > 0) fact *= (double)i;
        EXP_C[i] = (float)(1.0 / fact);
    }
    exp_ready = 1;
}

float oracle_expf(float x) {
    if (!exp_ready) exp_init();
    x = fminf(fmaxf(x, -87.0f), 88.0f);
    float n = rintf(x * EXP_LOG2E);
    float r = fmaf(-n, EXP_LN2_HI, x);
    r = fmaf(-n, EXP_LN2_LO, r);
    float p = EXP_C[7];
    for (int i = 6; i >= 0; --i) p = fmaf(p, r, EXP_C[i]);
    int32_t ni = (int32_t)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;
    float scale;
    memcpy(&scale, &bits, 4);
    return p * scale;
}

void oracle_expf_array(const float* x, int64_t n, float* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_expf(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Symmetric INT8 quantisation of one vector (per output channel for        */
/* weights, per token for activations): [MiniMax-M3 W8A8 on K100AI] s1.2,   */
/* s3.2.  scale = amax / 127 (fp32 division); q = rint(v / scale) with      */
/* ties to even, clamped to [-127, 127].  A scale that is 0 in fp32 (amax   */
/* == 0, or amax so small that amax / 127 underflows) gives q = 0.          */
/* ------------------------------------------------------------------------ */

static inline int8_t quant_one(float v, float scale) {
    float t = rintf(v / scale);
    if (t > 127.0f) t = 127.0f;
    if (t < -127.0f) t = -127.0f;
    return (int8_t)t;
}

/* Quantise n values read with a stride; writes q contiguously.  clip > 0    */
/* caps the range: amax = min(max |v|, clip), so values beyond the cap        */
/* saturate at +-127 instead of stretching the scale ([MiniMax-M3 W8A8 on     */
/* K100AI] s6.4, third defence: saturate at a threshold).                    */
static float quant_vector_clip(const float* v, int64_t n, int64_t stride, int8_t* q, float clip) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(v[i * stride]));
    if (clip > 0.0f && amax > clip) amax = clip;
    const float scale = amax / 127.0f;
    if (scale == 0.0f) {
        memset(q, 0, (size_t)n);
        return 0.0f;
    }
    for (int64_t i = 0; i < n; ++i) q[i] = quant_one(v[i * stride], scale);
    return scale;
}

static float quant_vector(const float* v, int64_t n, int64_t stride, int8_t* q) {
    return quant_vector_clip(v, n, stride, q, 0.0f);
}

void oracle_quantize_rows(const float* v, int64_t rows, int64_t n, int8_t* q, float* scale) {
    for (int64_t r = 0; r < rows; ++r) scale[r] = quant_vector(v + r * n, n, 1, q + r * n);
}

/* ------------------------------------------------------------------------ */
/* SmoothQuant ([MiniMax-M3 W8A8 on K100AI] s3.2, s6.1): move the outlier   */
/* difficulty of X into the weights with s_j = max|X_j|^a / max|W_j|^(1-a). */
/* ------------------------------------------------------------------------ */

/* Calibration statistic: per-channel max |x| over calibration rows. */
void oracle_channel_absmax(const float* x, int64_t rows, int32_t d, float* ax) {
    for (int32_t j = 0; j < d; ++j) ax[j] = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t j = 0; j < d; ++j) ax[j] = fmaxf(ax[j], fabsf(x[r * d + j]));
}

/* aw_j = max over experts e and output channels n of |W_gate[e][j][n]| and
 * |W_up[e][j][n]| (READING: one s per layer, because every expert's gate and
 * up projections read the same token activation).  Accumulates into aw, so
 * the experts may be passed in several chunks; aw must start at 0. */
void oracle_gateup_input_absmax(const float* w_gate, const float* w_up, int32_t n_experts,
                                int32_t d, int32_t f, float* aw) {
    for (int32_t e = 0; e < n_experts; ++e)
        for (int32_t j = 0; j < d; ++j) {
            const float* g = w_gate + ((int64_t)e * d + j) * f;
            const float* u = w_up + ((int64_t)e * d + j) * f;
            float m = aw[j];
            for (int32_t n = 0; n < f; ++n) {
                m = fmaxf(m, fabsf(g[n]));
                m = fmaxf(m, fabsf(u[n]));
            }
            aw[j] = m;
        }
}

/* s_j = fp32(ax^a / aw^(1-a)) evaluated in fp64 with both statistics floored
 * at 1e-5 (READING: avoids 0^a and division by zero); inv_s_j = fp32(1/s_j). */
void oracle_smooth_scales(const float* ax, const float* aw, int32_t d, float alpha,
                          float* s, float* inv_s) {
    double a = (double)alpha;
    for (int32_t j = 0; j < d; ++j) {
        double x = ax[j] > 1e-5f ? (double)ax[j] : (double)1e-5f;
        double w = aw[j] > 1e-5f ? (double)aw[j] : (double)1e-5f;
        s[j] = (float)(pow(x, a) / pow(w, 1.0 - a));
        inv_s[j] = (float)(1.0 / (double)s[j]);
    }
}

/* Gate or up weights of one expert, W [d][f] (input j, output n): smooth
 * each input row (W'[j][n] = fp32(s_j * W[j][n]); s may be NULL for no
 * smoothing) and quantise per output channel n over the d inputs.
 * Writes q [f][d] (output-channel major) and sw [f]. */
void oracle_quantize_gateup_expert(const float* w, const float* s, int32_t d, int32_t f,
                                   int8_t* q, float* sw) {
    float* col = (float*)malloc(sizeof(float) * (size_t)d);
    for (int32_t n = 0; n < f; ++n) {
        for (int32_t j = 0; j < d; ++j) {
            float v = w[(int64_t)j * f + n];
            col[j] = s ? s[j] * v : v;
        }
        sw[n] = quant_vector(col, d, 1, q + (int64_t)n * d);
    }
    free(col);
}

/* Down weights of one expert, W [f][d] (input j, output n), not smoothed
 * (READING: only the layer input X is smoothed); quantised per output
 * channel n over the f inputs.  Writes q [d][f] and sw [d]. */
void oracle_quantize_down_expert(const float* w, int32_t f, int32_t d, int8_t* q, float* sw) {
    for (int32_t n = 0; n < d; ++n) sw[n] = quant_vector(w + n, f, d, q + (int64_t)n * f);
}

/* ------------------------------------------------------------------------ */
/* Router ([Day0 adaptation] section 4: gate; top-k routing exact including */
/* the tie-break).                                                          */
/* ------------------------------------------------------------------------ */

/* Logit of token t for expert e, in a fixed fp32 order (READING): 32
 * partial sums, partial p = fmaf chain over i ascending of
 * x[32i+p] * W[32i+p][e] starting from +0; the partials are then combined
 * pairwise by distance 16, 8, 4, 2, 1 (p <- p + p^o) and partial 0 is the
 * logit.  W_router is [d][E].  d must be a multiple of 32. */
void oracle_router_logits(const float* x, const float* wr, int64_t T, int32_t d, int32_t E,
                          float* logits) {
    float* part = (float*)malloc(sizeof(float) * 32 * (size_t)E);
    float* next = (float*)malloc(sizeof(float) * 32 * (size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        const float* xt = x + t * d;
        for (int32_t p = 0; p < 32; ++p) {
            float* acc = part + (int64_t)p * E;
            for (int32_t e = 0; e < E; ++e) acc[e] = 0.0f;
            for (int32_t i = 0; i < d / 32; ++i) {
                int32_t j = 32 * i + p;
                float xv = xt[j];
                const float* w = wr + (int64_t)j * E;
                for (int32_t e = 0; e < E; ++e) acc[e] = fmaf(xv, w[e], acc[e]);
            }
        }
        for (int32_t o = 16; o >= 1; o >>= 1) {
            for (int32_t p = 0; p < 32; ++p)
                for (int32_t e = 0; e < E; ++e)
                    next[p * E + e] = part[p * E + e] + part[(p ^ o) * E + e];
            float* tmp = part; part = next; next = tmp;
        }
        for (int32_t e = 0; e < E; ++e) logits[t * E + e] = part[e];
    }
    free(part);
    free(next);
}

/* Top-k and gate weights.  l_e = logit + bias_e (bias may be NULL).  The k
 * experts taken are the first k in the order (l descending, e ascending):
 * equal logits go to the lower expert index.  Weights (READING: softmax over
 * the k selected logits, renormalised, when renormalize != 0; softmax over
 * all E otherwise): w_j = E(l_j - l_max) / Z, Z summed in slot order (or
 * expert order over all E), E = oracle_expf.  Slots are in rank order. */
void oracle_topk_softmax(const float* logits, const float* bias, int64_t T, int32_t E, int32_t k,
                         int32_t renormalize, int32_t* idx, float* w) {
    float* l = (float*)malloc(sizeof(float) * (size_t)E);
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) l[e] = bias ? logits[t * E + e] + bias[e] : logits[t * E + e];
        memset(taken, 0, (size_t)E);
        for (int32_t s = 0; s < k; ++s) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower index */
            }
            taken[best] = 1;
            idx[t * k + s] = best;
        }
        float lmax = l[idx[t * k]];
        if (renormalize) {
            float z = 0.0f;
            for (int32_t s = 0; s < k; ++s) z = z + oracle_expf(l[idx[t * k + s]] - lmax);
            for (int32_t s = 0; s < k; ++s) w[t * k + s] = oracle_expf(l[idx[t * k + s]] - lmax) / z;
        } else {
            float z = 0.0f;
            for (int32_t e = 0; e < E; ++e) z = z + oracle_expf(l[e] - lmax);
            for (int32_t s = 0; s < k; ++s) w[t * k + s] = oracle_expf(l[idx[t * k + s]] - lmax) / z;
        }
    }
    free(l);
    free(taken);
}

/* ------------------------------------------------------------------------ */
/* Capacity and permutation ([Day0 adaptation] section 4: sort / un-sort;   */
/* section 2 item 2: capacity factor, overflow dropped).                    */
/* ------------------------------------------------------------------------ */

/* C = ceil(cf * T * k / E) in fp64 (READING); cf <= 0 means no limit (-1).
 * No expert can receive more than T * k arrivals, so C is clamped to T * k
 * before the integer conversion: the kept set is the same, and a huge or
 * infinite cf no longer overflows the conversion. */
int32_t oracle_capacity(float cf, int64_t T, int32_t k, int32_t E) {
    if (!(cf > 0.0f)) return -1;
    const double tk = (double)(T * k);
    double c = ceil((double)cf * tk / (double)E);
    if (!(c <= tk)) c = tk;
    return (int32_t)c;
}

/* Rows are the kept (t, slot) pairs ordered by expert, then by token.  The
 * pairs are visited in token order, then slot order; an expert keeps its
 * first `cap` arrivals (cap < 0: all) and drops the rest (READING: dropped
 * slots contribute nothing and the kept weights are not renormalised).
 * Writes offsets [E+1] (exclusive scan of kept counts), row2ts [R] with
 * value t*k+slot, ts2row [T*k] (-1 for dropped).  Returns R. */
int32_t oracle_permute(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t cap,
                       int32_t* offsets, int32_t* row2ts, int32_t* ts2row) {
    int32_t* kept = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    unsigned char* keep = (unsigned char*)malloc((size_t)(T * k > 0 ? T * k : 1));
    for (int64_t i = 0; i < T * k; ++i) {
        int32_t e = idx[i];
        if (cap < 0 || kept[e] < cap) { kept[e]++; keep[i] = 1; }
        else keep[i] = 0;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + kept[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int64_t i = 0; i < T * k; ++i) {
        if (!keep[i]) { ts2row[i] = -1; continue; }
        int32_t e = idx[i];
        int32_t r = offsets[e] + fill[e]++;
        row2ts[r] = (int32_t)i;
        ts2row[i] = r;
    }
    int32_t R = offsets[E];
    free(kept);
    free(keep);
    free(fill);
    return R;
}

/* ------------------------------------------------------------------------ */
/* Per-token activation quantisation of the smoothed input                  */
/* ([MiniMax-M3 W8A8 on K100AI] s3.2, s6.4): x'_j = fp32(x_j * inv_s_j),    */
/* then the symmetric INT8 rule over the d channels of the token.           */
/* ------------------------------------------------------------------------ */
/* act_clip > 0: the token's range is capped at act_clip (saturation of the  */
/* smoothed values beyond it); 0: no cap.                                    */
void oracle_quantize_tokens(const float* x, const float* inv_s, int64_t T, int32_t d,
                            float act_clip, int8_t* q, float* sx) {
    float* xs = (float*)malloc(sizeof(float) * (size_t)d);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < d; ++j) xs[j] = inv_s ? x[t * d + j] * inv_s[j] : x[t * d + j];
        sx[t] = quant_vector_clip(xs, d, 1, q + t * d, act_clip);
    }
    free(xs);
}

/* ------------------------------------------------------------------------ */
/* Clip threshold from calibration data ("One night of MoE inference         */
/* optimisation", s3.2: the activation truncation percentile, 99.9; values   */
/* above that quantile of the activations' range are cut).  READING: the     */
/* percentile is taken over |x'| of every element of the calibration rows,   */
/* x' = fp32(x * inv_s) (the values the per-token quantiser sees), with the  */
/* nearest-rank rule: the ceil(p/100 * n)-th smallest value (p in (0, 100]). */
/* ------------------------------------------------------------------------ */
static int cmp_float(const void* a, const void* b) {
    const float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

float oracle_act_clip_percentile(const float* x, const float* inv_s, int64_t rows, int32_t d,
                                 double percent) {
    const int64_t n = rows * d;
    if (n <= 0) return 0.0f;
    float* a = (float*)malloc(sizeof(float) * (size_t)n);
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t j = 0; j < d; ++j) {
            const float v = inv_s ? x[r * d + j] * inv_s[j] : x[r * d + j];
            a[r * d + j] = fabsf(v);
        }
    qsort(a, (size_t)n, sizeof(float), cmp_float);
    int64_t rank = (int64_t)ceil(percent / 100.0 * (double)n);
    if (rank < 1) rank = 1;
    if (rank > n) rank = n;
    const float c = a[rank - 1];
    free(a);
    return c;
}

/* ------------------------------------------------------------------------ */
/* INT8 x INT8 -> INT32 GEMM: c[m][n] = sum_k a[m][k] * b[n][k]             */
/* ([MiniMax-M3 W8A8 on K100AI] s1.2).  Exact: |c| <= 127^2 K < 2^31.       */
/* ------------------------------------------------------------------------ */
void oracle_gemm_i8(const int8_t* a, const int8_t* b, int64_t M, int64_t N, int64_t K, int32_t* c) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t acc = 0;
            const int8_t* ar = a + m * K;
            const int8_t* br = b + n * K;
            for (int64_t kk = 0; kk < K; ++kk) acc += (int32_t)ar[kk] * (int32_t)br[kk];
            c[m * N + n] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* Expert FFN epilogues.                                                    */
/* ------------------------------------------------------------------------ */

/* Dequantise gate and up, SwiGLU, and requantise h per row (the expert's
 * intermediate stays INT8 between the two matmuls: [MiniMax-M3 W8A8 on
 * K100AI] s4.3).  g = fp32(fp32(acc_g * sx) * sw_g), likewise u;
 * silu(g) = g / (1 + E(-g)); h = silu(g) * u; then the INT8 rule over the f
 * values of the row.  h_out may be NULL. */
void oracle_swiglu_requant(const int32_t* acc_g, const int32_t* acc_u, float sx,
                           const float* sw_g, const float* sw_u, int32_t f,
                           float* h_out, int8_t* hq, float* sh) {
    float* h = (float*)malloc(sizeof(float) * (size_t)f);
    for (int32_t n = 0; n < f; ++n) {
        float g = ((float)acc_g[n] * sx) * sw_g[n];
        float u = ((float)acc_u[n] * sx) * sw_u[n];
        float silu = g / (1.0f + oracle_expf(-g));
        h[n] = silu * u;
    }
    if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)f);
    *sh = quant_vector(h, f, 1, hq);
    free(h);
}

/* Down projection epilogue: o = fp32(fp32(fp32(acc2 * sh) * sw_dn) * w). */
void oracle_down_epilogue(const int32_t* acc2, float sh, const float* sw_dn, float w, int32_t d,
                          float* o) {
    for (int32_t n = 0; n < d; ++n) o[n] = (((float)acc2[n] * sh) * sw_dn[n]) * w;
}

/* fp32 -> bf16 (nearest even) and back, for the bf16 output. */
float oracle_round_bf16(float v) {
    uint32_t b;
    memcpy(&b, &v, 4);
    b += 0x7FFFu + ((b >> 16) & 1u);
    b &= 0xFFFF0000u;
    memcpy(&v, &b, 4);
    return v;
}

/* ------------------------------------------------------------------------ */
/* The whole layer for a list of tokens ([Day0 adaptation] section 4: gate, */
/* sort, grouped expert GEMMs, un-sort, weighted sum).                      */
/* ------------------------------------------------------------------------ */

/*
 * Inputs: x [T][d] fp32 values; quantised weights in the oracle's layout
 * (wq_gate, wq_up [E][f][d] with sw_gate, sw_up [E][f]; wq_down [E][d][f]
 * with sw_down [E][d]); inv_s [d] (NULL: no smoothing); act_clip (0: none,
 * else the cap of the per-token range, see oracle_quantize_tokens); routing already
 * done (idx, w [T][k]; ts2row [T][k], -1 = dropped).  Computes the tokens
 * listed in tok[n_sel].  Outputs per selected token i: y [i][d] (fp32 sum
 * y = ((0 + o_slot0) + o_slot1) + ... over kept slots, then bf16-rounded if
 * out_bf16), and per (i, slot): acc1 [i][s][2f] (gate | up), hq [i][s][f],
 * sh [i][s], acc2 [i][s][d], o [i][s][d].  Any debug output may be NULL.
 * Also xq [i][d], sx [i].
 * READING ([Day0 adaptation] section 4 un-sorts the expert outputs and then
 * forms the weighted sum, without fixing the precision of the per-slot rows
 * in between): for a bf16-output layer each per-slot row o is stored in the
 * layer's output precision, bf16 (nearest even), before the slot-order sum;
 * an fp32-output layer keeps it in fp32.
 */
void oracle_moe_tokens(const float* x, int32_t d, int32_t f, int32_t E, int32_t k,
                       const int8_t* wq_gate, const int8_t* wq_up, const float* sw_gate,
                       const float* sw_up, const int8_t* wq_down, const float* sw_down,
                       const float* inv_s, float act_clip, const int32_t* idx, const float* w,
                       const int32_t* ts2row, const int64_t* tok, int64_t n_sel, int32_t out_bf16,
                       float* y, int8_t* xq_out, float* sx_out, int32_t* acc1_out, int8_t* hq_out,
                       float* sh_out, int32_t* acc2_out, float* o_out) {
    (void)E;
    int8_t* xq = (int8_t*)malloc((size_t)d);
    int32_t* acc_g = (int32_t*)malloc(sizeof(int32_t) * (size_t)f);
    int32_t* acc_u = (int32_t*)malloc(sizeof(int32_t) * (size_t)f);
    int8_t* hq = (int8_t*)malloc((size_t)f);
    int32_t* acc2 = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
    float* o = (float*)malloc(sizeof(float) * (size_t)d);
    for (int64_t i = 0; i < n_sel; ++i) {
        int64_t t = tok[i];
        float sx;
        oracle_quantize_tokens(x + t * d, inv_s, 1, d, act_clip, xq, &sx);
        if (xq_out) memcpy(xq_out + i * d, xq, (size_t)d);
        if (sx_out) sx_out[i] = sx;
        float* yt = y + i * d;
        for (int32_t n = 0; n < d; ++n) yt[n] = 0.0f;
        for (int32_t s = 0; s < k; ++s) {
            int64_t ts = t * k + s;
            int32_t e = idx[ts];
            int64_t dbg = i * k + s;
            if (ts2row[ts] < 0) {
                if (sh_out) sh_out[dbg] = 0.0f;
                continue;
            }
            oracle_gemm_i8(xq, wq_gate + (int64_t)e * f * d, 1, f, d, acc_g);
            oracle_gemm_i8(xq, wq_up + (int64_t)e * f * d, 1, f, d, acc_u);
            float sh;
            oracle_swiglu_requant(acc_g, acc_u, sx, sw_gate + (int64_t)e * f, sw_up + (int64_t)e * f,
                                  f, NULL, hq, &sh);
            oracle_gemm_i8(hq, wq_down + (int64_t)e * d * f, 1, d, f, acc2);
            oracle_down_epilogue(acc2, sh, sw_down + (int64_t)e * d, w[ts], d, o);
            if (out_bf16)
                for (int32_t n = 0; n < d; ++n) o[n] = oracle_round_bf16(o[n]);
            for (int32_t n = 0; n < d; ++n) yt[n] = yt[n] + o[n];
            if (acc1_out) {
                memcpy(acc1_out + dbg * 2 * f, acc_g, sizeof(int32_t) * (size_t)f);
                memcpy(acc1_out + dbg * 2 * f + f, acc_u, sizeof(int32_t) * (size_t)f);
            }
            if (hq_out) memcpy(hq_out + dbg * f, hq, (size_t)f);
            if (sh_out) sh_out[dbg] = sh;
            if (acc2_out) memcpy(acc2_out + dbg * d, acc2, sizeof(int32_t) * (size_t)d);
            if (o_out) memcpy(o_out + dbg * d, o, sizeof(float) * (size_t)d);
        }
        if (out_bf16)
            for (int32_t n = 0; n < d; ++n) yt[n] = oracle_round_bf16(yt[n]);
    }
    free(xq); free(acc_g); free(acc_u); free(hq); free(acc2); free(o);
}

/* ======================================================================== */
/* FP8 (E4M3) experts ([Day0 adaptation] section 1: expert layers stored in  */
/* FP8 or INT8, with the activations kept on the same precision path as the  */
/* weights; the deployment config names FP8 experts).                        */
/* ======================================================================== */

/*
 * E4M3, the finite-only 8-bit float of the OCP FP8 formats: 1 sign bit, 4
 * exponent bits (bias 7), 3 mantissa bits, no infinities; exponent 1111 with
 * mantissa 111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
 * Normal values (8 + m) 2^(e-10) for e = 1..15, subnormals m 2^-9.
 * READING: rounding is to the nearest representable value, ties to the even
 * code; magnitudes beyond 448 saturate to 448 (a finite input never becomes
 * NaN); the sign is kept, so tiny negative values give -0 (code 0x80).
 */

/* Spacing of E4M3 values in the binade of a (0 < a < 448). */
static float e4m3_step(float a) {
    int e;
    frexpf(a, &e);            /* a = m 2^e, m in [0.5, 1): binade 2^(e-1) */
    int be = e - 1;
    if (be < -6) be = -6;     /* the subnormals share the lowest binade's spacing */
    return ldexpf(1.0f, be - 3);
}

/* The E4M3 value nearest to v (as a float). */
float oracle_e4m3_round(float v) {
    float a = fabsf(v);
    float r;
    if (a >= 448.0f) {
        r = 448.0f;
    } else if (a == 0.0f) {
        r = 0.0f;
    } else {
        const float q = e4m3_step(a);
        r = rintf(a / q) * q;  /* a / q is exact (q is a power of two) */
        if (r > 448.0f) r = 448.0f;
    }
    return signbit(v) ? -r : r;
}

uint8_t oracle_e4m3_encode(float v) {
    const float r = fabsf(oracle_e4m3_round(v));
    const uint8_t s = signbit(v) ? 0x80 : 0x00;
    if (r == 0.0f) return s;
    int e;
    frexpf(r, &e);
    const int be = e - 1;
    if (be < -6) return (uint8_t)(s | (int)(r / ldexpf(1.0f, -9)));          /* subnormal */
    const int m = (int)(r / ldexpf(1.0f, be - 3)) - 8;
    return (uint8_t)(s | ((be + 7) << 3) | m);
}

float oracle_e4m3_decode(uint8_t c) {
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float a;
    if (e == 15 && m == 7) a = NAN;
    else if (e == 0) a = ldexpf((float)m, -9);
    else a = ldexpf((float)(8 + m), e - 10);
    return s ? -a : a;
}

void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* q) {
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_array(const uint8_t* q, int64_t n, float* v) {
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e4m3_decode(q[i]);
}

/* Scaled E4M3 quantisation of one vector (the FP8 counterpart of the INT8   */
/* rule): scale = amax / 448 (fp32 division), q = e4m3(v / scale); a scale  */
/* that is 0 in fp32 gives codes 0; clip > 0 caps amax as in the INT8 rule.  */
static float quant_vector_fp8(const float* v, int64_t n, int64_t stride, uint8_t* q, float clip) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(v[i * stride]));
    if (clip > 0.0f && amax > clip) amax = clip;
    const float scale = amax / 448.0f;
    if (scale == 0.0f) {   /* amax == 0, or amax / 448 underflows: codes 0 */
        memset(q, 0, (size_t)n);
        return 0.0f;
    }
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i * stride] / scale);
    return scale;
}

void oracle_quantize_rows_fp8(const float* v, int64_t rows, int64_t n, uint8_t* q, float* scale) {
    for (int64_t r = 0; r < rows; ++r) scale[r] = quant_vector_fp8(v + r * n, n, 1, q + r * n, 0.0f);
}

/* Expert weights in E4M3, per output channel, as the INT8 quantisers above:  */
/* gate/up from w [d][f] with the smoothing fold (q [f][d]), down from        */
/* w [f][d] without it (q [d][f]).                                            */
void oracle_quantize_gateup_expert_fp8(const float* w, const float* s, int32_t d, int32_t f, uint8_t* q,
                                       float* sw) {
    float* col = (float*)malloc(sizeof(float) * (size_t)d);
    for (int32_t n = 0; n < f; ++n) {
        for (int32_t j = 0; j < d; ++j) col[j] = s ? s[j] * w[(int64_t)j * f + n] : w[(int64_t)j * f + n];
        sw[n] = quant_vector_fp8(col, d, 1, q + (int64_t)n * d, 0.0f);
    }
    free(col);
}

void oracle_quantize_down_expert_fp8(const float* w, int32_t f, int32_t d, uint8_t* q, float* sw) {
    for (int32_t n = 0; n < d; ++n) sw[n] = quant_vector_fp8(w + n, f, d, q + (int64_t)n * f, 0.0f);
}

void oracle_quantize_tokens_fp8(const float* x, const float* inv_s, int64_t T, int32_t d, float act_clip,
                                uint8_t* q, float* sx) {
    float* xs = (float*)malloc(sizeof(float) * (size_t)d);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < d; ++j) xs[j] = inv_s ? x[t * d + j] * inv_s[j] : x[t * d + j];
        sx[t] = quant_vector_fp8(xs, d, 1, q + t * d, act_clip);
    }
    free(xs);
}

/* E4M3 x E4M3 GEMM, c[m][n] = sum_k a[m][k] b[n][k], computed exactly and  */
/* rounded once to fp32.  Exact in fp64: every product of two E4M3 values is */
/* a multiple of 2^-18 below 2^18, so a sum of up to 2^16 of them needs at   */
/* most 52 significant bits.                                                 */
void oracle_gemm_fp8(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N, int64_t K, float* c) {
    double lut[256];
    for (int i = 0; i < 256; ++i) lut[i] = (double)oracle_e4m3_decode((uint8_t)i);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            const uint8_t* ar = a + m * K;
            const uint8_t* br = b + n * K;
            for (int64_t kk = 0; kk < K; ++kk) acc += lut[ar[kk]] * lut[br[kk]];
            c[m * N + n] = (float)acc;
        }
}

/* SwiGLU on the fp32 accumulators of the FP8 path, then E4M3 per row. */
void oracle_swiglu_requant_fp8(const float* acc_g, const float* acc_u, float sx, const float* sw_g,
                               const float* sw_u, int32_t f, float* h_out, uint8_t* hq, float* sh) {
    float* h = (float*)malloc(sizeof(float) * (size_t)f);
    for (int32_t n = 0; n < f; ++n) {
        float g = (acc_g[n] * sx) * sw_g[n];
        float u = (acc_u[n] * sx) * sw_u[n];
        float silu = g / (1.0f + oracle_expf(-g));
        h[n] = silu * u;
    }
    if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)f);
    *sh = quant_vector_fp8(h, f, 1, hq, 0.0f);
    free(h);
}

/* The whole layer with FP8 experts: as oracle_moe_tokens, with E4M3 codes   */
/* (uint8) for weights, tokens and h, and fp32 accumulators.                 */
void oracle_moe_tokens_fp8(const float* x, int32_t d, int32_t f, int32_t E, int32_t k,
                           const uint8_t* wq_gate, const uint8_t* wq_up, const float* sw_gate,
                           const float* sw_up, const uint8_t* wq_down, const float* sw_down,
                           const float* inv_s, float act_clip, const int32_t* idx, const float* w,
                           const int32_t* ts2row, const int64_t* tok, int64_t n_sel, int32_t out_bf16,
                           float* y, uint8_t* xq_out, float* sx_out, float* acc1_out, uint8_t* hq_out,
                           float* sh_out, float* acc2_out, float* o_out) {
    (void)E;
    uint8_t* xq = (uint8_t*)malloc((size_t)d);
    float* acc_g = (float*)malloc(sizeof(float) * (size_t)f);
    float* acc_u = (float*)malloc(sizeof(float) * (size_t)f);
    uint8_t* hq = (uint8_t*)malloc((size_t)f);
    float* acc2 = (float*)malloc(sizeof(float) * (size_t)d);
    float* o = (float*)malloc(sizeof(float) * (size_t)d);
    for (int64_t i = 0; i < n_sel; ++i) {
        const int64_t t = tok[i];
        float sx;
        oracle_quantize_tokens_fp8(x + t * d, inv_s, 1, d, act_clip, xq, &sx);
        if (xq_out) memcpy(xq_out + i * d, xq, (size_t)d);
        if (sx_out) sx_out[i] = sx;
        float* yt = y + i * d;
        for (int32_t n = 0; n < d; ++n) yt[n] = 0.0f;
        for (int32_t s = 0; s < k; ++s) {
            const int64_t ts = t * k + s;
            const int32_t e = idx[ts];
            const int64_t dbg = i * k + s;
            if (ts2row[ts] < 0) {
                if (sh_out) sh_out[dbg] = 0.0f;
                continue;
            }
            oracle_gemm_fp8(xq, wq_gate + (int64_t)e * f * d, 1, f, d, acc_g);
            oracle_gemm_fp8(xq, wq_up + (int64_t)e * f * d, 1, f, d, acc_u);
            float sh;
            oracle_swiglu_requant_fp8(acc_g, acc_u, sx, sw_gate + (int64_t)e * f, sw_up + (int64_t)e * f, f,
                                      NULL, hq, &sh);
            oracle_gemm_fp8(hq, wq_down + (int64_t)e * d * f, 1, d, f, acc2);
            for (int32_t n = 0; n < d; ++n) o[n] = ((acc2[n] * sh) * sw_down[(int64_t)e * d + n]) * w[ts];
            if (out_bf16)   /* per-slot rows in the output precision, as for INT8 experts */
                for (int32_t n = 0; n < d; ++n) o[n] = oracle_round_bf16(o[n]);
            for (int32_t n = 0; n < d; ++n) yt[n] = yt[n] + o[n];
            if (acc1_out) {
                memcpy(acc1_out + dbg * 2 * f, acc_g, sizeof(float) * (size_t)f);
                memcpy(acc1_out + dbg * 2 * f + f, acc_u, sizeof(float) * (size_t)f);
            }
            if (hq_out) memcpy(hq_out + dbg * f, hq, (size_t)f);
            if (sh_out) sh_out[dbg] = sh;
            if (acc2_out) memcpy(acc2_out + dbg * d, acc2, sizeof(float) * (size_t)d);
            if (o_out) memcpy(o_out + dbg * d, o, sizeof(float) * (size_t)d);
        }
        if (out_bf16)
            for (int32_t n = 0; n < d; ++n) yt[n] = oracle_round_bf16(yt[n]);
    }
    free(xq); free(acc_g); free(acc_u); free(hq); free(acc2); free(o);
}
