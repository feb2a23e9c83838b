/*
 * CPU oracle for the sparse MoE layer forward pass — TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct C in fp64.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg load this library; the product path
 * (the CUDA library) shares no code, header or table with it.
 *
 * What it computes, step by step, in the order the pages give the layer
 * ("Expert Parallelism" guide (infra.bea.ai), section 2 "The Dispatch
 * Pattern"; "Expert Parallelism" glossary (klaylearn.com), third paragraph):
 *   1. router logits  l[t,e] = sum_i x[t,i] * Wr[i,e] (+ bias[e]); the router
 *      is a linear scoring layer with one output per expert
 *        (inferensys.com glossary, gating-network and router-latency entries)
 *   2. top-k gating: the k experts with the largest logits, ties to the lower
 *      expert index; gate weights = softmax over the k selected logits
 *        (inferensys.com glossary, Top-k Gating; klaylearn.com glossary: the
 *         router also yields the weights that mix the expert outputs)
 *   3. capacity C = ceil(cf*k*T/E), dropless (C = T) when cf == 0
 *        (inferensys.com glossary, capacity-factor entry; "Expert Parallelism
 *         & All-to-All" (neelmishra), section "Why fixed-size buffers matter
 *         here")
 *   4. permutation into per-expert buckets: pairs take bucket slots in token
 *      order; a pair whose slot is >= C overflows a full bucket and is dropped
 *        (inferensys.com glossary, Dropped Tokens entry)
 *   5. per-expert SwiGLU MLP: h = silu(x Wg) * (x Wu), o = h Wd
 *        (neelmishra, section "Tensor parallelism for experts": gate, up and
 *         down projections).  The expert GEMMs take bf16 operands, so h, the
 *        down projection's input, is rounded to bf16 (nearest, ties to even)
 *        before o = h Wd when round_h is set; with round_h clear the whole
 *        MLP stays in fp64.
 *   6. combine: y[t] = sum over kept pairs of w * o, in the token's top-k
 *      order; a token whose every pair was dropped leaves the layer as it came
 *        (neelmishra, section "All-to-all: the distributed transpose": the
 *         combine undoes the dispatch permutation and sums the k outputs
 *         scaled by their gate weights; inferensys.com glossary, Dropped
 *         Tokens entry: a dropped token goes through the layer untouched)
 *
 * The FP8 variant of step 5 (e4m3 weights with one fp32 scale per expert
 * column, e4m3 activations with one fp32 scale per row; inferensys.com
 * glossary, quantization entry) is defined further down with its own rule.
 *
 * bf16 tensors are passed as their raw 16-bit patterns (uint16_t) and are
 * widened exactly to double.  All accumulation is fp64.  Layouts are
 * row-major: x[T,d], Wr[d,E], Wg/Wu[E,d,f], Wd[E,f,d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the calling host thread's parallel regions use from now on (a
 * per-thread setting: a test that calls the oracle from several host threads
 * at once gives each a share of the cores).  No effect on any result. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Step 3.  cf == 0 selects the dropless layer: an expert can receive each
 * token at most once, so C = T never drops.  Evaluated as ((cf*k)*T)/E in
 * fp64, then rounded up. */
int64_t oracle_capacity(int64_t T, int64_t E, int64_t k, double cf) {
    if (cf == 0.0) return T;
    double c = ((cf * (double)k) * (double)T) / (double)E;
    return (int64_t)ceil(c);
}

/* Step 1, fp64 accumulation.  bias may be NULL. */
void oracle_router_logits(const uint16_t* x, const float* w_router, const float* bias,
                          int64_t T, int64_t d, int64_t E, double* logits) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i)
                acc += bf16_bits_to_f64(x[t * d + i]) * (double)w_router[i * E + e];
            if (bias) acc += (double)bias[e];
            logits[t * E + e] = acc;
        }
    }
}

/* Step 2 on fp32 logits (the precision the routing decision is taken in).
 * Repeated selection of the largest remaining logit; a strict '>' keeps the
 * lower expert index on ties.  Output order: descending logit.  Weights:
 * exp(l_j - l_max) / sum over the k selected, in fp64. */
void oracle_topk(const float* logits, int64_t T, int64_t E, int64_t k,
                 int32_t* topk_idx, double* topk_w) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            topk_idx[t * k + j] = (int32_t)best;
        }
        free(taken);
        double lmax = (double)l[topk_idx[t * k]];
        double sum = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            double v = exp((double)l[topk_idx[t * k + j]] - lmax);
            topk_w[t * k + j] = v;
            sum += v;
        }
        for (int64_t j = 0; j < k; ++j) topk_w[t * k + j] /= sum;
    }
}

/* Step 4.  Walk tokens in index order; each (token, expert) pair takes the
 * next free slot of its expert's bucket; slot >= C means dropped (slot = -1).
 * counts[e] = pairs kept by e, offsets = exclusive prefix sum of counts
 * (offsets[E] = N kept pairs), row_src[offsets[e] + slot] = t for kept pairs.
 * Returns the number of dropped pairs. */
int64_t oracle_permute(const int32_t* topk_idx, int64_t T, int64_t E, int64_t k, int64_t C,
                       int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* row_src) {
    int64_t* demand = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < k; ++j) {
            int64_t e = topk_idx[t * k + j];
            int64_t s = demand[e]++;
            slot[t * k + j] = (s < C) ? (int32_t)s : -1;
        }
    }
    int64_t n_drop = 0, run = 0;
    for (int64_t e = 0; e < E; ++e) {
        int64_t kept = demand[e] < C ? demand[e] : C;
        counts[e] = (int32_t)kept;
        offsets[e] = (int32_t)run;
        run += kept;
        n_drop += demand[e] - kept;
    }
    offsets[E] = (int32_t)run;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < k; ++j) {
            int32_t s = slot[t * k + j];
            if (s >= 0) row_src[offsets[topk_idx[t * k + j]] + s] = (int32_t)t;
        }
    free(demand);
    return n_drop;
}

/* The gather half of step 4: row r of the permuted buffer is token row_src[r]. */
void oracle_dispatch(const uint16_t* x, const int32_t* row_src, int64_t N, int64_t d,
                     uint16_t* x_perm) {
    for (int64_t r = 0; r < N; ++r)
        memcpy(x_perm + r * d, x + (int64_t)row_src[r] * d, (size_t)d * sizeof(uint16_t));
}

/* Round a finite double in the normal bf16 range to the nearest bf16 value
 * (8 significant bits), ties to even: scale the mantissa to [128, 256) and
 * round it to an integer in the default round-half-even mode. */
double oracle_round_bf16(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int ex;
    double m = frexp(v, &ex);            /* v = m * 2^ex, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8));
    return ldexp(r, ex - 8);
}

/* Step 5 for n rows that all go to one expert whose weights are wg/wu [d,f]
 * and wd [f,d].  h [n,f] (may be NULL) and o [n,d] in fp64; h is rounded to
 * bf16 before the down projection when round_h != 0.
 * silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
void oracle_swiglu_rows(const uint16_t* x_rows, int64_t n, int64_t d, int64_t f,
                        const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                        int round_h, double* h_out, double* o_out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double* g = (double*)calloc((size_t)f, sizeof(double));
        double* u = (double*)calloc((size_t)f, sizeof(double));
        const uint16_t* xr = x_rows + r * d;
        for (int64_t i = 0; i < d; ++i) {
            double xi = bf16_bits_to_f64(xr[i]);
            const uint16_t* wgi = wg + i * f;
            const uint16_t* wui = wu + i * f;
            for (int64_t j = 0; j < f; ++j) {
                g[j] += xi * bf16_bits_to_f64(wgi[j]);
                u[j] += xi * bf16_bits_to_f64(wui[j]);
            }
        }
        double* o = o_out + r * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t j = 0; j < f; ++j) {
            double hj = g[j] / (1.0 + exp(-g[j])) * u[j];
            if (round_h) hj = oracle_round_bf16(hj);
            if (h_out) h_out[r * f + j] = hj;
            const uint16_t* wdj = wd + j * d;
            for (int64_t c = 0; c < d; ++c) o[c] += hj * bf16_bits_to_f64(wdj[c]);
        }
        free(g);
        free(u);
    }
}

/* ---- The padded [E, C, d] layout (a variant of step 4's buffer) ----
 * Fixed-size expert buffers ("Expert Parallelism & All-to-All" (neelmishra),
 * section "Why fixed-size buffers matter here"): bucket e occupies rows
 * e*C .. e*C + C - 1; a kept pair (t, j) of expert e with slot s puts x[t] at
 * row e*C + s; rows past a bucket's count stay zero.  row_src gives each
 * row's token, -1 on padding rows. */
void oracle_dispatch_padded(const uint16_t* x, const int32_t* topk_idx, const int32_t* slot,
                            int64_t T, int64_t d, int64_t k, int64_t E, int64_t C, uint16_t* out,
                            int32_t* row_src) {
    memset(out, 0, (size_t)(E * C * d) * sizeof(uint16_t));
    for (int64_t r = 0; r < E * C; ++r) row_src[r] = -1;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < k; ++j) {
            const int64_t s = slot[t * k + j];
            if (s < 0) continue;
            const int64_t row = (int64_t)topk_idx[t * k + j] * C + s;
            memcpy(out + row * d, x + t * d, (size_t)d * sizeof(uint16_t));
            row_src[row] = (int32_t)t;
        }
}

/* ---- FP8 (e4m3) expert weights: one variant of step 5's operands ----
 * Weight-only quantization with one scale per (expert, output column):
 *   s[e,n] = max_k |w[e,k,n]| / 448   (fp32, as the quantizer computes it)
 *   q[e,k,n] = e4m3(w[e,k,n] / s[e,n]) (the fp32 quotient rounded to the
 *             nearest e4m3 value, ties to even; 448 is the largest finite)
 * and the dequantized weight q * s used in place of w.  e4m3: 1 sign bit,
 * 4 exponent bits (bias 7), 3 mantissa bits; normal values 2^-6 .. 448,
 * subnormals k * 2^-9. */

/* nearest e4m3 code (ties to even) of a finite float, saturating to +-448 */
unsigned char oracle_e4m3_encode(float v) {
    unsigned char sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;                 /* 1.75 * 2^8 */
    if (a < ldexp(1.0, -6)) {                            /* subnormal range: k * 2^-9 */
        double k = nearbyint(a * 512.0);                 /* ties to even */
        if (k >= 8.0) return sign | 0x08;                /* rounds up to 2^-6 */
        return sign | (unsigned char)k;
    }
    int ex;
    double m = frexp(a, &ex);                            /* a = m * 2^ex, 0.5 <= m < 1 */
    double r = nearbyint(ldexp(m, 4));                   /* 4 significant bits: 8..16 */
    if (r >= 16.0) { r = 8.0; ex += 1; }
    int e = ex - 1 + 7;                                  /* biased exponent of r/8 * 2^(ex-1) */
    if (e > 15 || (e == 15 && r > 14.0)) return sign | 0x7E;
    return sign | (unsigned char)((e << 3) | ((int)r - 8));
}

double oracle_e4m3_decode(unsigned char q) {
    int e = (q >> 3) & 0xF, m = q & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (q & 0x80) ? -v : v;
}

/* Quantize bf16 weights [E,K,N] to e4m3 codes + fp32 column scales [E,N]. */
void oracle_quantize_fp8(const uint16_t* w, int64_t E, int64_t K, int64_t N, unsigned char* q,
                         float* scale) {
    for (int64_t e = 0; e < E; ++e)
        for (int64_t n = 0; n < N; ++n) {
            float mx = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float a = fabsf((float)bf16_bits_to_f64(w[(e * K + k) * N + n]));
                if (a > mx) mx = a;
            }
            float s = mx > 0.0f ? mx / 448.0f : 1.0f;
            scale[e * N + n] = s;
            for (int64_t k = 0; k < K; ++k) {
                float v = (float)bf16_bits_to_f64(w[(e * K + k) * N + n]) / s;
                q[(e * K + k) * N + n] = oracle_e4m3_encode(v);
            }
        }
}

/* Dequantized weights q * s as fp64 [E,K,N]. */
void oracle_dequant_fp8(const unsigned char* q, const float* scale, int64_t E, int64_t K,
                        int64_t N, double* out) {
    for (int64_t e = 0; e < E; ++e)
        for (int64_t k = 0; k < K; ++k)
            for (int64_t n = 0; n < N; ++n)
                out[(e * K + k) * N + n] =
                    oracle_e4m3_decode(q[(e * K + k) * N + n]) * (double)scale[e * N + n];
}

/* Step 5 for n rows of one expert with fp64 weights wg/wu [d,f], wd [f,d]
 * (e.g. dequantized FP8); otherwise as oracle_swiglu_rows. */
void oracle_swiglu_rows_f64w(const uint16_t* x_rows, int64_t n, int64_t d, int64_t f,
                             const double* wg, const double* wu, const double* wd, int round_h,
                             double* h_out, double* o_out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double* g = (double*)calloc((size_t)f, sizeof(double));
        double* u = (double*)calloc((size_t)f, sizeof(double));
        const uint16_t* xr = x_rows + r * d;
        for (int64_t i = 0; i < d; ++i) {
            double xi = bf16_bits_to_f64(xr[i]);
            for (int64_t j = 0; j < f; ++j) {
                g[j] += xi * wg[i * f + j];
                u[j] += xi * wu[i * f + j];
            }
        }
        double* o = o_out + r * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t j = 0; j < f; ++j) {
            double hj = g[j] / (1.0 + exp(-g[j])) * u[j];
            if (round_h) hj = oracle_round_bf16(hj);
            if (h_out) h_out[r * f + j] = hj;
            for (int64_t c = 0; c < d; ++c) o[c] += hj * wd[j * d + c];
        }
        free(g);
        free(u);
    }
}

/* ---- FP8 weights and activations (the W8A8 variant of step 5) ----
 * Activations are quantized per row with the same rule as the weight
 * columns above: s[r] = max_k |x[r,k]| / 448 (fp32; 1 for an all-zero row),
 * q[r,k] = e4m3(x[r,k] / s[r]).  A product of a row scale and a column scale
 * is constant along the contraction, so the quantized GEMM is
 *   out[r,n] = sum_k (q_a[r,k] s_a[r]) (q_w[k,n] s_w[n])
 * evaluated here on the dequantized operands in fp64. */
void oracle_quantize_rows_fp8(const uint16_t* x, int64_t R, int64_t K, unsigned char* q,
                              float* scale) {
    for (int64_t r = 0; r < R; ++r) {
        float mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf((float)bf16_bits_to_f64(x[r * K + k]));
            if (a > mx) mx = a;
        }
        float s = mx > 0.0f ? mx / 448.0f : 1.0f;
        scale[r] = s;
        for (int64_t k = 0; k < K; ++k)
            q[r * K + k] = oracle_e4m3_encode((float)bf16_bits_to_f64(x[r * K + k]) / s);
    }
}

/* Dequantized rows q * s as fp64 [R,K]. */
void oracle_dequant_rows_fp8(const unsigned char* q, const float* scale, int64_t R, int64_t K,
                             double* out) {
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = oracle_e4m3_decode(q[r * K + k]) * (double)scale[r];
}

/* Gate/up of one expert on fp64 operands: h = silu(a wg) * (a wu) for a [n,d],
 * wg/wu [d,f]; h rounded to bf16 when round_h is set. */
void oracle_gate_up_f64(const double* a, int64_t n, int64_t d, int64_t f, const double* wg,
                        const double* wu, int round_h, double* h_out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double* g = (double*)calloc((size_t)f, sizeof(double));
        double* u = (double*)calloc((size_t)f, sizeof(double));
        for (int64_t i = 0; i < d; ++i) {
            double ai = a[r * d + i];
            for (int64_t j = 0; j < f; ++j) {
                g[j] += ai * wg[i * f + j];
                u[j] += ai * wu[i * f + j];
            }
        }
        for (int64_t j = 0; j < f; ++j) {
            double hj = g[j] / (1.0 + exp(-g[j])) * u[j];
            h_out[r * f + j] = round_h ? oracle_round_bf16(hj) : hj;
        }
        free(g);
        free(u);
    }
}

/* out[n,N] = a[n,K] w[K,N] in fp64. */
void oracle_matmul_f64(const double* a, int64_t n, int64_t K, const double* w, int64_t N,
                       double* out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double* o = out + r * N;
        for (int64_t c = 0; c < N; ++c) o[c] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double ak = a[r * K + k];
            for (int64_t c = 0; c < N; ++c) o[c] += ak * w[k * N + c];
        }
    }
}

/* Step 5 over every bucket: rows offsets[e] .. offsets[e+1]-1 use expert e. */
void oracle_expert_mlp(const uint16_t* x_perm, const int32_t* offsets, int64_t E, int64_t d,
                       int64_t f, const uint16_t* w_gate, const uint16_t* w_up,
                       const uint16_t* w_down, int round_h, double* h, double* y_perm) {
    for (int64_t e = 0; e < E; ++e) {
        int64_t r0 = offsets[e], n = offsets[e + 1] - offsets[e];
        if (n == 0) continue;
        oracle_swiglu_rows(x_perm + r0 * d, n, d, f, w_gate + e * d * f, w_up + e * d * f,
                           w_down + e * f * d, round_h, h ? h + r0 * f : NULL, y_perm + r0 * d);
    }
}

/* Step 6.  Sum in the token's top-k order; a token with no kept pair returns
 * its input row. */
void oracle_combine(const double* y_perm, const uint16_t* x, const int32_t* topk_idx,
                    const double* topk_w, const int32_t* slot, const int32_t* offsets,
                    int64_t T, int64_t d, int64_t k, double* y) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* yt = y + t * d;
        int kept = 0;
        for (int64_t c = 0; c < d; ++c) yt[c] = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            int32_t s = slot[t * k + j];
            if (s < 0) continue;
            kept = 1;
            const double* o = y_perm + ((int64_t)offsets[topk_idx[t * k + j]] + s) * d;
            double w = topk_w[t * k + j];
            for (int64_t c = 0; c < d; ++c) yt[c] += w * o[c];
        }
        if (!kept)
            for (int64_t c = 0; c < d; ++c) yt[c] = bf16_bits_to_f64(x[t * d + c]);
    }
}

/* Steps 1-6 end to end (round_h as in step 5).  decision_logits (fp32 [T,E]) may be given, in which
 * case the routing decision is taken on those values; when NULL the oracle's
 * own fp64 logits, rounded to fp32, are used.  Optional outputs (NULL to skip):
 * logits64 [T,E], topk_idx [T,k], topk_w [T,k], slot [T,k], counts [E],
 * offsets [E+1].  Returns the number of dropped pairs. */
int64_t oracle_moe_forward(const uint16_t* x, const float* w_router, const float* bias,
                           const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                           int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf,
                           int round_h, const float* decision_logits, double* y,
                           double* logits64_out,
                           int32_t* topk_idx_out, double* topk_w_out, int32_t* slot_out,
                           int32_t* counts_out, int32_t* offsets_out) {
    double* l64 = (double*)malloc((size_t)(T * E) * sizeof(double));
    float* l32 = (float*)malloc((size_t)(T * E) * sizeof(float));
    int32_t* idx = (int32_t*)malloc((size_t)(T * k) * sizeof(int32_t));
    double* w = (double*)malloc((size_t)(T * k) * sizeof(double));
    int32_t* slot = (int32_t*)malloc((size_t)(T * k) * sizeof(int32_t));
    int32_t* counts = (int32_t*)malloc((size_t)E * sizeof(int32_t));
    int32_t* offsets = (int32_t*)malloc((size_t)(E + 1) * sizeof(int32_t));
    int32_t* row_src = (int32_t*)malloc((size_t)(T * k) * sizeof(int32_t));

    oracle_router_logits(x, w_router, bias, T, d, E, l64);
    if (decision_logits) {
        memcpy(l32, decision_logits, (size_t)(T * E) * sizeof(float));
    } else {
        for (int64_t i = 0; i < T * E; ++i) l32[i] = (float)l64[i];
    }
    oracle_topk(l32, T, E, k, idx, w);
    int64_t C = oracle_capacity(T, E, k, cf);
    int64_t n_drop = oracle_permute(idx, T, E, k, C, counts, offsets, slot, row_src);
    int64_t N = offsets[E];
    uint16_t* x_perm = (uint16_t*)malloc((size_t)(N * d + 1) * sizeof(uint16_t));
    double* y_perm = (double*)malloc((size_t)(N * d + 1) * sizeof(double));
    oracle_dispatch(x, row_src, N, d, x_perm);
    oracle_expert_mlp(x_perm, offsets, E, d, f, w_gate, w_up, w_down, round_h, NULL, y_perm);
    oracle_combine(y_perm, x, idx, w, slot, offsets, T, d, k, y);

    if (logits64_out) memcpy(logits64_out, l64, (size_t)(T * E) * sizeof(double));
    if (topk_idx_out) memcpy(topk_idx_out, idx, (size_t)(T * k) * sizeof(int32_t));
    if (topk_w_out) memcpy(topk_w_out, w, (size_t)(T * k) * sizeof(double));
    if (slot_out) memcpy(slot_out, slot, (size_t)(T * k) * sizeof(int32_t));
    if (counts_out) memcpy(counts_out, counts, (size_t)E * sizeof(int32_t));
    if (offsets_out) memcpy(offsets_out, offsets, (size_t)(E + 1) * sizeof(int32_t));
    free(l64); free(l32); free(idx); free(w); free(slot); free(counts); free(offsets);
    free(row_src); free(x_perm); free(y_perm);
    return n_drop;
}
