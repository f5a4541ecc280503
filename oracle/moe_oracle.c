/* moe_oracle.c -- plain FP64 CPU oracle of the fused MoE layer forward.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT (see moe_oracle.h for the
 * sources, the readings and who may call it).  Deliberately simple: loops in
 * the order the definitions are written, OpenMP only across independent
 * tokens / rows / groups, no blocking, no fusion.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math: the
 * FP8 code decisions below depend on IEEE single-precision division).
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------
 * Formats.
 * bfloat16: sign, 8 exponent bits (bias 127), 7 stored mantissa bits; the
 * upper half of an IEEE binary32 word.
 * e4m3 (OCP 8-bit floating point, "E4M3"): sign, 4 exponent bits (bias 7),
 * 3 mantissa bits, subnormals at exponent field 0, no infinities, the only
 * NaN patterns S.1111.111; largest finite magnitude 1.75 * 2^8 = 448.
 * ------------------------------------------------------------------------- */

double orc_bf16_decode(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* nearest multiple of 2^qe, ties to even (default rounding mode) */
static double round_to_quantum(double a, int qe) {
    return ldexp(nearbyint(ldexp(a, -qe)), qe);
}

uint16_t orc_bf16_round(double v) {
    if (isnan(v)) return 0x7fc0;
    double a = fabs(v);
    uint16_t sgn = signbit(v) ? 0x8000 : 0;
    if (a == 0.0) return sgn;
    int e;
    frexp(a, &e);                       /* a in [2^(e-1), 2^e)              */
    int qe = e - 8;                     /* 8 significant bits               */
    if (qe < -133) qe = -133;           /* subnormal spacing 2^-126 * 2^-7  */
    double r = isinf(a) ? a : round_to_quantum(a, qe);
    float f = (float)r;                 /* exact: r is on the bf16 grid, or
                                           rounds up past the top -> inf    */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sgn | (u >> 16));
}

void orc_bf16_round_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_round(v[i]);
}

double orc_e4m3_decode(uint8_t b) {
    int s = b >> 7, E = (b >> 3) & 15, M = b & 7;
    if (E == 15 && M == 7) return NAN;
    double v = (E == 0) ? ldexp((double)M, -9)             /* M/8 * 2^-6      */
                        : ldexp((double)(8 + M), E - 10);   /* (1+M/8)*2^(E-7) */
    return s ? -v : v;
}

uint8_t orc_e4m3_round(double v) {
    if (isnan(v)) return 0x7f;
    uint8_t sgn = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    if (a == 0.0) return sgn;
    double r;
    if (isinf(a)) {
        r = 448.0;
    } else {
        int e;
        frexp(a, &e);                   /* a in [2^(e-1), 2^e)              */
        int qe = e - 4;                 /* 4 significant bits               */
        if (qe < -9) qe = -9;           /* subnormal spacing 2^-6 * 2^-3    */
        r = round_to_quantum(a, qe);
        if (r > 448.0) r = 448.0;       /* saturate to the largest finite   */
    }
    if (r == 0.0) return sgn;
    if (r < ldexp(1.0, -6)) return (uint8_t)(sgn | (int)ldexp(r, 9));
    int e;
    frexp(r, &e);                       /* r in [2^(e-1), 2^e): exponent e-1 */
    int M = (int)ldexp(r, 4 - e) - 8;   /* r / 2^(e-1) * 8 - 8, in 0..7     */
    return (uint8_t)(sgn | ((e - 1 + 7) << 3) | M);
}

/* One quantisation group: s = fp32(amax) / 448 in FP32 (amax == 0 -> 1),
 * q_i = e4m3(fp32(v_i / s)).  The divisions are single precision on purpose:
 * the kernel takes the same decision in the same precision. */
static float quant_group(const float* v, int n, int64_t stride, uint8_t* q, int64_t qstride) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[(int64_t)i * stride]);
        if (a > amax) amax = a;
    }
    volatile float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
    for (int i = 0; i < n; ++i) {
        volatile float t = v[(int64_t)i * stride] / s;
        q[(int64_t)i * qstride] = orc_e4m3_round((double)t);
    }
    return s;
}

/* ---------------------------------------------------------------------------
 * Per-tensor FP8: one scale per weight matrix; static activation scales
 * ------------------------------------------------------------------------- */

void orc_quant_fp8_tensor(const uint16_t* W, int64_t batch, int rows, int cols, uint8_t* q,
                          float* s) {
    int64_t n = (int64_t)rows * cols;
    #pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < batch; ++b) {
        float* f = (float*)malloc(sizeof(float) * (size_t)n);
        for (int64_t i = 0; i < n; ++i) f[i] = (float)orc_bf16_decode(W[b * n + i]);
        s[b] = quant_group(f, (int)n, 1, q + b * n, 1);
        free(f);
    }
}

void orc_quant_fp8_static(const float* v, int64_t n, float s, uint8_t* q) {
    for (int64_t i = 0; i < n; ++i) {
        volatile float t = v[i] / s;
        q[i] = orc_e4m3_round((double)t);
    }
}

/* ---------------------------------------------------------------------------
 * [MX] MXFP8: E8M0 shared scale per block of 32, e4m3 elements
 * ------------------------------------------------------------------------- */

double orc_e8m0_decode(uint8_t b) {
    if (b == 255) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* shared_exp = floor(log2(amax)) - 8, clamped to [-127, 127] (amax == 0 ->
 * -127); the byte is shared_exp + 127. */
uint8_t orc_mx_scale_byte(float amax) {
    if (!(amax > 0.0f)) return 0;
    int e;
    frexp((double)amax, &e);            /* amax in [2^(e-1), 2^e)           */
    int se = (e - 1) - 8;
    if (se < -127) se = -127;
    if (se > 127) se = 127;
    return (uint8_t)(se + 127);
}

static void quant_mx_block(const float* v, int n, uint8_t* q, uint8_t* sb) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    uint8_t b = orc_mx_scale_byte(amax);
    double X = orc_e8m0_decode(b);
    for (int i = 0; i < n; ++i) q[i] = orc_e4m3_round((double)v[i] / X);
    *sb = b;
}

void orc_quant_mx_rows(const float* v, int64_t rows, int cols, uint8_t* q, uint8_t* s) {
    int g = cols / 32;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < g; ++j)
            quant_mx_block(v + r * cols + j * 32, 32, q + r * cols + j * 32, s + r * g + j);
}

void orc_quant_mx_bf16(const uint16_t* W, int64_t batch, int rows, int cols, uint8_t* q,
                       uint8_t* s) {
    int64_t n = batch * rows;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        float f[32];
        for (int j = 0; j < cols / 32; ++j) {
            for (int i = 0; i < 32; ++i) f[i] = (float)orc_bf16_decode(W[r * cols + j * 32 + i]);
            quant_mx_block(f, 32, q + r * cols + j * 32, s + r * (cols / 32) + j);
        }
    }
}

/* ---------------------------------------------------------------------------
 * [RG] router split and logits
 * ------------------------------------------------------------------------- */

void orc_router_split(const float* W, int64_t n, uint16_t* hi, uint16_t* lo) {
    for (int64_t i = 0; i < n; ++i) {
        double w = (double)W[i];
        uint16_t h = orc_bf16_round(w);
        double r = w - orc_bf16_decode(h);   /* exact: both are binary32    */
        hi[i] = h;
        lo[i] = orc_bf16_round(r * 256.0);   /* low part stored times 256   */
    }
}

void orc_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                       const float* bias, int T, int d, int E, double* logits) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) {
                double w = orc_bf16_decode(hi[(int64_t)e * d + i]) +
                           orc_bf16_decode(lo[(int64_t)e * d + i]) / 256.0;
                acc += orc_bf16_decode(x[(int64_t)t * d + i]) * w;
            }
            if (bias) acc += (double)bias[e];
            logits[(int64_t)t * E + e] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * [FM][HY] top-k routing
 * ------------------------------------------------------------------------- */

void orc_route_topk(const float* logits, int T, int E, int k, int renorm,
                    int32_t* ids, double* w) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        /* k rounds of "largest remaining, lowest id on ties" == a full sort
           by (value descending, id ascending) cut after k entries */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            ids[(int64_t)t * k + j] = best;
        }
        double lmax = (double)l[ids[(int64_t)t * k]];
        double denom = 0.0;
        if (renorm) {
            for (int j = 0; j < k; ++j) denom += exp((double)l[ids[(int64_t)t * k + j]] - lmax);
        } else {
            for (int e = 0; e < E; ++e) denom += exp((double)l[e] - lmax);
        }
        for (int j = 0; j < k; ++j)
            w[(int64_t)t * k + j] = exp((double)l[ids[(int64_t)t * k + j]] - lmax) / denom;
        free(taken);
    }
}

/* ---------------------------------------------------------------------------
 * [FP] per-expert counts, contiguous intervals, stable permutation
 * ------------------------------------------------------------------------- */

void orc_permute(const int32_t* ids, int T, int E, int k, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* inv) {
    int64_t n = (int64_t)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < n; ++a) counts[ids[a]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t a = 0; a < n; ++a) {
        int32_t p = cursor[ids[a]]++;
        perm[p] = (int32_t)a;
        inv[a] = p;
    }
    free(cursor);
}

/* ---------------------------------------------------------------------------
 * [G8][HY] FP8 quantisation
 * ------------------------------------------------------------------------- */

void orc_quant_fp8_blocks(const uint16_t* W, int64_t batch, int rows, int cols,
                          uint8_t* q, float* s) {
    int rb = rows / 128, cb = cols / 128;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t blk = 0; blk < batch * rb * cb; ++blk) {
        int64_t b = blk / ((int64_t)rb * cb);
        int r0 = (int)((blk / cb) % rb) * 128, c0 = (int)(blk % cb) * 128;
        float* v = (float*)malloc(sizeof(float) * 128 * 128);
        uint8_t* qq = (uint8_t*)malloc(128 * 128);
        for (int r = 0; r < 128; ++r)
            for (int c = 0; c < 128; ++c)
                v[r * 128 + c] = (float)orc_bf16_decode(W[(b * rows + r0 + r) * (int64_t)cols + c0 + c]);
        s[blk] = quant_group(v, 128 * 128, 1, qq, 1);
        for (int r = 0; r < 128; ++r)
            memcpy(q + (b * rows + r0 + r) * (int64_t)cols + c0, qq + r * 128, 128);
        free(v);
        free(qq);
    }
}

void orc_quant_fp8_rows(const float* v, int64_t rows, int cols, uint8_t* q, float* s) {
    int g = cols / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < g; ++j)
            s[r * g + j] = quant_group(v + r * cols + j * 128, 128, 1, q + r * cols + j * 128, 1);
}

/* ---------------------------------------------------------------------------
 * Expert FFN stages
 * ------------------------------------------------------------------------- */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Dense weights of one group, decoded to FP64 ([rows][cols]); FP8 layers use
 * the oracle's own 128x128 block quantisation of the BF16 weights. */
static double* group_weights(const orc_layer* L, const uint16_t* W, int rows, int cols) {
    int64_t n = (int64_t)rows * cols;
    double* out = (double*)malloc(sizeof(double) * (size_t)n);
    if (L->wdtype == 0) {
        for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_decode(W[i]);
        return out;
    }
    if (L->wdtype == 3) {
        uint8_t* q = (uint8_t*)malloc((size_t)n);
        float sw;
        orc_quant_fp8_tensor(W, 1, rows, cols, q, &sw);
        for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(q[i]) * (double)sw;
        free(q);
        return out;
    }
    if (L->wdtype == 2) {
        uint8_t* q = (uint8_t*)malloc((size_t)n);
        uint8_t* sb = (uint8_t*)malloc((size_t)(n / 32 + 1));
        orc_quant_mx_bf16(W, 1, rows, cols, q, sb);
        for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(q[i]) * orc_e8m0_decode(sb[i / 32]);
        free(q);
        free(sb);
        return out;
    }
    int rb = rows / 128, cb = cols / 128;
    uint8_t* q = (uint8_t*)malloc((size_t)n);
    float* s = (float*)malloc(sizeof(float) * (size_t)rb * cb);
    orc_quant_fp8_blocks(W, 1, rows, cols, q, s);
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            out[(int64_t)r * cols + c] =
                orc_e4m3_decode(q[(int64_t)r * cols + c]) * (double)s[(r / 128) * cb + c / 128];
    free(q);
    free(s);
    return out;
}

/* An activation row as the GEMM consumes it: BF16 values as they are, or for
 * FP8 layers the dequantised 1x128-group quantisation of the FP32 row. */
static void activation_row(const orc_layer* L, const double* v, int n, double* out,
                           float static_scale) {
    if (L->wdtype == 0) {
        for (int i = 0; i < n; ++i) out[i] = v[i];
        return;
    }
    float* f = (float*)malloc(sizeof(float) * (size_t)n);
    uint8_t* q = (uint8_t*)malloc((size_t)n);
    for (int i = 0; i < n; ++i) f[i] = (float)v[i];
    if (L->wdtype == 3) {
        orc_quant_fp8_static(f, n, static_scale, q);
        for (int i = 0; i < n; ++i) out[i] = orc_e4m3_decode(q[i]) * (double)static_scale;
        free(f);
        free(q);
        return;
    }
    if (L->wdtype == 2) {
        uint8_t* sb = (uint8_t*)malloc((size_t)(n / 32 + 1));
        orc_quant_mx_rows(f, 1, n, q, sb);
        for (int i = 0; i < n; ++i) out[i] = orc_e4m3_decode(q[i]) * orc_e8m0_decode(sb[i / 32]);
        free(f);
        free(q);
        free(sb);
        return;
    }
    float* s = (float*)malloc(sizeof(float) * (size_t)(n / 128));
    orc_quant_fp8_rows(f, 1, n, q, s);
    for (int i = 0; i < n; ++i) out[i] = orc_e4m3_decode(q[i]) * (double)s[i / 128];
    free(f);
    free(q);
    free(s);
}

static int64_t total_rows(const orc_layer* L) {
    return (int64_t)L->T * L->k + (L->Is > 0 ? L->T : 0);
}

void orc_gateup(const orc_layer* L, const uint16_t* x, const int32_t* perm,
                const int32_t* offsets, double* h) {
    int d = L->d, hs = L->I > L->Is ? L->I : L->Is;
    int ngroups = L->E + (L->Is > 0 ? 1 : 0);
    int64_t Tk = (int64_t)L->T * L->k;
    #pragma omp parallel for schedule(dynamic)
    for (int g = 0; g < ngroups; ++g) {
        int64_t p0 = g < L->E ? offsets[g] : Tk;
        int64_t p1 = g < L->E ? offsets[g + 1] : Tk + L->T;
        if (p1 <= p0) continue;
        int I = g < L->E ? L->I : L->Is;
        const uint16_t* Wsrc = g < L->E ? L->w_gu + (int64_t)g * 2 * I * d : L->ws_gu;
        double* W = group_weights(L, Wsrc, 2 * I, d);
        double* xr = (double*)malloc(sizeof(double) * (size_t)d);
        double* xa = (double*)malloc(sizeof(double) * (size_t)d);
        for (int64_t p = p0; p < p1; ++p) {
            int64_t t = g < L->E ? perm[p] / L->k : p - Tk;
            for (int i = 0; i < d; ++i) xr[i] = orc_bf16_decode(x[t * d + i]);
            activation_row(L, xr, d, xa, L->act_sx);
            for (int n = 0; n < I; ++n) {
                double gs = 0.0, us = 0.0;
                const double* wg = W + (int64_t)n * d;
                const double* wu = W + (int64_t)(I + n) * d;
                for (int i = 0; i < d; ++i) {
                    gs += xa[i] * wg[i];
                    us += xa[i] * wu[i];
                }
                h[p * hs + n] = silu(gs) * us;
            }
        }
        free(W);
        free(xr);
        free(xa);
    }
}

void orc_down(const orc_layer* L, const double* h, const int32_t* offsets, double* o) {
    int d = L->d, hs = L->I > L->Is ? L->I : L->Is;
    int ngroups = L->E + (L->Is > 0 ? 1 : 0);
    int64_t Tk = (int64_t)L->T * L->k;
    #pragma omp parallel for schedule(dynamic)
    for (int g = 0; g < ngroups; ++g) {
        int64_t p0 = g < L->E ? offsets[g] : Tk;
        int64_t p1 = g < L->E ? offsets[g + 1] : Tk + L->T;
        if (p1 <= p0) continue;
        int I = g < L->E ? L->I : L->Is;
        const uint16_t* Wsrc = g < L->E ? L->w_d + (int64_t)g * d * I : L->ws_d;
        double* W = group_weights(L, Wsrc, d, I);
        double* ha = (double*)malloc(sizeof(double) * (size_t)I);
        for (int64_t p = p0; p < p1; ++p) {
            activation_row(L, h + p * hs, I, ha, L->act_sh);
            for (int n = 0; n < d; ++n) {
                double acc = 0.0;
                const double* w = W + (int64_t)n * I;
                for (int i = 0; i < I; ++i) acc += ha[i] * w[i];
                o[p * d + n] = acc;
            }
        }
        free(W);
        free(ha);
    }
}

void orc_combine(const orc_layer* L, const double* o, const int32_t* inv,
                 const double* w, double* y) {
    int d = L->d, k = L->k;
    int64_t Tk = (int64_t)L->T * k;
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < L->T; ++t) {
        for (int n = 0; n < d; ++n) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(int64_t)t * k + j] * o[(int64_t)inv[(int64_t)t * k + j] * d + n];
            if (L->Is > 0) acc += o[(Tk + t) * d + n];
            y[(int64_t)t * d + n] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * The whole layer: router logits -> top-k -> permute -> gate-up -> down ->
 * combine.  Routing is decided on the FP32 rounding of the FP64 logits.
 * ------------------------------------------------------------------------- */

int orc_forward(const orc_layer* L, const uint16_t* x, orc_out* out) {
    int T = L->T, d = L->d, E = L->E, k = L->k;
    int64_t Tk = (int64_t)T * k, R = total_rows(L);
    int hs = L->I > L->Is ? L->I : L->Is;
    uint16_t* hi = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)E * d);
    uint16_t* lo = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)E * d);
    double* logits = (double*)malloc(sizeof(double) * (size_t)T * E);
    float* logits32 = (float*)malloc(sizeof(float) * (size_t)T * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)Tk);
    double* w = (double*)malloc(sizeof(double) * (size_t)Tk);
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)Tk);
    int32_t* inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)Tk);
    double* h = (double*)calloc((size_t)R * hs, sizeof(double));
    double* o = (double*)calloc((size_t)R * d, sizeof(double));
    if (!hi || !lo || !logits || !logits32 || !ids || !w || !counts || !offsets ||
        !perm || !inv || !h || !o)
        return 1;

    orc_router_split(L->router_w, (int64_t)E * d, hi, lo);
    orc_router_logits(x, hi, lo, L->router_bias, T, d, E, logits);
    for (int64_t i = 0; i < (int64_t)T * E; ++i) logits32[i] = (float)logits[i];
    orc_route_topk(logits32, T, E, k, L->renorm, ids, w);
    orc_permute(ids, T, E, k, counts, offsets, perm, inv);
    orc_gateup(L, x, perm, offsets, h);
    orc_down(L, h, offsets, o);
    orc_combine(L, o, inv, w, out->y);

    if (out->logits) memcpy(out->logits, logits, sizeof(double) * (size_t)T * E);
    if (out->ids) memcpy(out->ids, ids, sizeof(int32_t) * (size_t)Tk);
    if (out->w) memcpy(out->w, w, sizeof(double) * (size_t)Tk);
    if (out->counts) memcpy(out->counts, counts, sizeof(int32_t) * (size_t)E);
    if (out->offsets) memcpy(out->offsets, offsets, sizeof(int32_t) * (size_t)(E + 1));
    if (out->perm) memcpy(out->perm, perm, sizeof(int32_t) * (size_t)Tk);
    if (out->inv) memcpy(out->inv, inv, sizeof(int32_t) * (size_t)Tk);
    free(hi); free(lo); free(logits); free(logits32); free(ids); free(w);
    free(counts); free(offsets); free(perm); free(inv); free(h); free(o);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Fused all-reduce + residual + RMSNorm (tensor parallelism)
 * ------------------------------------------------------------------------- */

void orc_allreduce_rmsnorm(const uint16_t* x, int G, int T, int d, const uint16_t* residual,
                           const uint16_t* gamma, double eps, double* res, double* out) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) {
            double s = residual ? orc_bf16_decode(residual[(int64_t)t * d + i]) : 0.0;
            for (int r = 0; r < G; ++r) s += orc_bf16_decode(x[((int64_t)r * T + t) * d + i]);
            res[(int64_t)t * d + i] = s;
            ss += s * s;
        }
        const double inv = 1.0 / sqrt(ss / d + eps);
        for (int i = 0; i < d; ++i)
            out[(int64_t)t * d + i] = res[(int64_t)t * d + i] * inv * orc_bf16_decode(gamma[i]);
    }
}
