/*
 * Reference oracle for the QoQ W4A8 path: progressive group quantization of
 * the weights, per-token INT8 quantization of the activations, the exact
 * integer GEMM and the FP16 output scaling.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is plain, slow, obviously-correct C.
 * It shares no code, header, table or constant generator with the CUDA
 * library, and the library never calls it.  Only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark load it.
 *
 * Sources (the method is described in prose only):
 *  - "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
 *    Serving" (velog notes), Methods, 1) Algorithm: QoQ -- weights are first
 *    quantized to 8 bits with per-channel FP16 scales, and the 8-bit
 *    intermediate is quantized again to 4 bits, so that every GEMM runs on
 *    INT8 tensor cores.
 *  - same page, Methods, 2) System: QServe -- the "protective range" of the
 *    first level lets the 4-bit to 8-bit dequantization run with
 *    register-level parallelism, computed as "subtraction after
 *    multiplication": dq = q*s2 - z*s2.
 *  - same page, Background -- per-group W4A4 has to dequantize INT32 partial
 *    sums inside the main loop; W4A8 with a per-channel first level does not,
 *    so the FP16 scaling is applied once, after the whole K reduction.
 *  - "Part5 LLM部署技术", 3. 实践扩展：QServe（W4A8KV4） -- kernel fusion that
 *    avoids dequantizing partial sums.
 *  - The concrete numeric format implemented here: symmetric per-channel
 *    INT8 weights with FP16 scales, groups of 128 (or 64) input channels,
 *    asymmetric UINT4 codes with INT8 group scales and UINT4 zeros,
 *    per-token symmetric INT8 activations with FP16 scales, INT32
 *    accumulation.  The pages name these pieces only in words.
 *
 * Readings taken where the pages are silent:
 *  - protective range R1 = 119 for the first level;
 *  - s2 = max(1, ceil((max - min) / 15)) with the group range widened to
 *    include 0; z = round_half_even(-min / s2);
 *  - round half to even everywhere; the FP16-rounded scale is the one used
 *    for the division, which is done in IEEE binary32 (the kernel's
 *    precision), so that both sides take every integer decision alike;
 *  - a scale that would round to 0 in FP16 becomes 1 for an all-zero row and
 *    the smallest positive FP16 value otherwise;
 *  - the output Y = fp16(acc * sx * s1) is formed here in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_R1 119      /* protective range of the first (per-channel) level */
#define ORC_QMAX_X 127  /* symmetric per-token activation range */

/* ---------------------------------------------------------------------------
 * IEEE 754 binary16 conversions, written from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * ------------------------------------------------------------------------- */

double orc_h2d(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);            /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

float orc_h2f(uint16_t h) { return (float)orc_h2d(h); }

/* Round to nearest, ties to even, of a non-negative double that is an
 * integer plus a fraction. */
static double round_half_even_d(double n) {
    double fl = floor(n);
    double diff = n - fl;
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* binary64 -> binary16, round to nearest even (one rounding step). */
uint16_t orc_d2h(double x) {
    uint16_t sign = (uint16_t)(signbit(x) ? 0x8000 : 0);
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    /* 65520 is half-way between the largest finite value (65504) and 2^16;
     * the tie goes to the even neighbour, which is 2^16, i.e. infinity. */
    if (a >= 65520.0) return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; a result of 1024 quanta encodes
         * the smallest normal number, which is also the right bit pattern */
        double n = round_half_even_d(ldexp(a, 24));
        return sign | (uint16_t)n;
    }
    int e;
    (void)frexp(a, &e);        /* a = m * 2^e with m in [0.5, 1) */
    e -= 1;                    /* a = (1.f) * 2^e */
    double n = round_half_even_d(ldexp(a, 10 - e)); /* in [1024, 2048] */
    if (n == 2048.0) { n = 1024.0; e += 1; }
    int biased = e + 15;
    if (biased >= 31) return sign | 0x7c00;
    return sign | (uint16_t)((biased << 10) | ((int)n - 1024));
}

uint16_t orc_f2h(float x) { return orc_d2h((double)x); }

/* Array forms, for exhaustive checks. */
void orc_h2d_array(const uint16_t* h, long n, double* out) {
    for (long i = 0; i < n; ++i) out[i] = orc_h2d(h[i]);
}
void orc_f2h_array(const float* x, long n, uint16_t* out) {
    for (long i = 0; i < n; ++i) out[i] = orc_f2h(x[i]);
}
void orc_d2h_array(const double* x, long n, uint16_t* out) {
    for (long i = 0; i < n; ++i) out[i] = orc_d2h(x[i]);
}

/* ---------------------------------------------------------------------------
 * Rounding helpers for the integer decisions.
 * ------------------------------------------------------------------------- */

/* Round half to even of a binary32 value (the C library's rintf in the
 * default rounding mode). */
static float rne_f(float v) { return rintf(v); }

/* Exact round-half-even of the rational a/b with b > 0, in integers. */
int orc_rne_div(int a, int b) {
    int q = a / b;                 /* truncates toward zero */
    int r = a - q * b;             /* same sign as a */
    if (r < 0) { r = -r; }
    int twice = 2 * r;
    if (twice > b || (twice == b && (q & 1))) {
        q += (a < 0) ? -1 : 1;
    }
    return q;
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* FP16 scale = amax / qmax rounded to FP16; guarded against 0. */
static uint16_t scale_from_absmax(float amax, float qmax) {
    if (amax == 0.0f) return 0x3c00;             /* 1.0 */
    uint16_t s = orc_f2h(amax / qmax);
    if ((s & 0x7fff) == 0) s = 0x0001;           /* smallest positive FP16 */
    return s;
}

/* ---------------------------------------------------------------------------
 * Level 1 of progressive group quantization: per output channel, symmetric
 * INT8 with an FP16 scale, limited to the protective range [-119, 119].
 * W is N x K row-major FP16 (the [out, in] layout of a linear layer).
 * ------------------------------------------------------------------------- */
void orc_quant_w_level1(const uint16_t* W, int N, int K,
                        uint16_t* s1, int8_t* W8) {
    for (int n = 0; n < N; ++n) {
        const uint16_t* row = W + (size_t)n * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float v = fabsf(orc_h2f(row[k]));
            if (v > amax) amax = v;
        }
        uint16_t s = scale_from_absmax(amax, (float)ORC_R1);
        s1[n] = s;
        float sf = orc_h2f(s);
        for (int k = 0; k < K; ++k) {
            float t = orc_h2f(row[k]) / sf;      /* IEEE binary32 division */
            int v = (int)rne_f(t);
            W8[(size_t)n * K + k] = (int8_t)clampi(v, -ORC_R1, ORC_R1);
        }
    }
}

/* ---------------------------------------------------------------------------
 * Level 2: each group of G consecutive input channels of the INT8
 * intermediate becomes asymmetric UINT4 codes q with an INT8 scale s2 and a
 * UINT4 zero z, so that dq = (q - z) * s2 = q*s2 - z*s2.
 * q is N x K (one code per byte), s2 and z are N x (K/G).
 * ------------------------------------------------------------------------- */
void orc_quant_w_level2(const int8_t* W8, int N, int K, int G,
                        uint8_t* q, int8_t* s2, uint8_t* z) {
    int ng = K / G;
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            const int8_t* w = W8 + (size_t)n * K + (size_t)g * G;
            int mn = 0, mx = 0;                  /* range always holds 0 */
            for (int i = 0; i < G; ++i) {
                if (w[i] < mn) mn = w[i];
                if (w[i] > mx) mx = w[i];
            }
            int range = mx - mn;
            int s = (range + 14) / 15;           /* ceil(range / 15) */
            if (s < 1) s = 1;
            int zz = orc_rne_div(-mn, s);
            s2[(size_t)n * ng + g] = (int8_t)s;
            z[(size_t)n * ng + g] = (uint8_t)zz;
            for (int i = 0; i < G; ++i) {
                int c = orc_rne_div(w[i], s) + zz;
                q[(size_t)n * K + (size_t)g * G + i] = (uint8_t)clampi(c, 0, 15);
            }
        }
    }
}

/* dq = q*s2 - z*s2: the INT8 operand the tensor cores consume. */
void orc_dequant_w(const uint8_t* q, const int8_t* s2, const uint8_t* z,
                   int N, int K, int G, int8_t* dq) {
    int ng = K / G;
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            int s = s2[(size_t)n * ng + k / G];
            int zz = z[(size_t)n * ng + k / G];
            int v = (int)q[(size_t)n * K + k] * s - zz * s;
            dq[(size_t)n * K + k] = (int8_t)v;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Per-token symmetric INT8 activations with an FP16 scale per row.
 * X is M x K row-major FP16.
 * ------------------------------------------------------------------------- */
void orc_quant_act(const uint16_t* X, int M, int K, uint16_t* sx, int8_t* X8) {
    for (int m = 0; m < M; ++m) {
        const uint16_t* row = X + (size_t)m * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float v = fabsf(orc_h2f(row[k]));
            if (v > amax) amax = v;
        }
        uint16_t s = scale_from_absmax(amax, (float)ORC_QMAX_X);
        sx[m] = s;
        float sf = orc_h2f(s);
        for (int k = 0; k < K; ++k) {
            int v = (int)rne_f(orc_h2f(row[k]) / sf);
            X8[(size_t)m * K + k] = (int8_t)clampi(v, -ORC_QMAX_X, ORC_QMAX_X);
        }
    }
}

/* ---------------------------------------------------------------------------
 * acc[m, n] = sum_k X8[m, k] * dq[n, k], exactly (int64, then checked to fit
 * INT32).  Returns the number of entries that did not fit INT32.
 * ------------------------------------------------------------------------- */
int64_t orc_dot_i8(const int8_t* a, const int8_t* b, int K) {
    int64_t s = 0;
    for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
    return s;
}

long orc_int_gemm(const int8_t* X8, const int8_t* dq, int M, int N, int K,
                  int32_t* acc) {
    long overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : overflow)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            int64_t s = orc_dot_i8(X8 + (size_t)m * K, dq + (size_t)n * K, K);
            if (s > INT32_MAX || s < INT32_MIN) overflow += 1;
            acc[(size_t)m * N + n] = (int32_t)s;
        }
    }
    return overflow;
}

/* The same sum for a list of (m, n) positions only. */
void orc_int_gemm_at(const int8_t* X8, const int8_t* dq, int K,
                     const int64_t* ms, const int64_t* ns, long count,
                     int64_t* out) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        out[i] = orc_dot_i8(X8 + (size_t)ms[i] * K, dq + (size_t)ns[i] * K, K);
    }
}

/* ---------------------------------------------------------------------------
 * Output scaling, applied once after the whole K reduction:
 * Y[m, n] = fp16(acc[m, n] * sx[m] * s1[n]), formed in binary64.
 * ------------------------------------------------------------------------- */
void orc_epilogue(const int32_t* acc, const uint16_t* sx, const uint16_t* s1,
                  int M, int N, uint16_t* Y) {
    for (int m = 0; m < M; ++m) {
        double a = orc_h2d(sx[m]);
        for (int n = 0; n < N; ++n) {
            double v = (double)acc[(size_t)m * N + n] * a * orc_h2d(s1[n]);
            Y[(size_t)m * N + n] = orc_d2h(v);
        }
    }
}

/* Whole online path for one layer: activations -> INT8, GEMM, scaling. */
long orc_w4a8_forward(const uint16_t* X, const int8_t* dq, const uint16_t* s1,
                      int M, int N, int K, int8_t* X8, uint16_t* sx,
                      int32_t* acc, uint16_t* Y) {
    orc_quant_act(X, M, K, sx, X8);
    long of = orc_int_gemm(X8, dq, M, N, K, acc);
    orc_epilogue(acc, sx, s1, M, N, Y);
    return of;
}

/* ---------------------------------------------------------------------------
 * Per-input-channel smoothing, SmoothQuant style ("Part5 LLM部署技术",
 * 1.1 权重-激活联合量化：SmoothQuant): part of the activations' quantization
 * difficulty is moved onto the weights, one factor per input channel k.
 *  1. calibration: the per-channel maxima of the activations (over a
 *     calibration batch) and of the weights;
 *  2. smoothing: the activations are divided by the factor, the weights
 *     multiplied by it, so X . W^T is unchanged up to rounding;
 *  3. inference: the smoothed operands are quantized as usual.
 * Readings where the page's formula is lost: migration strength alpha = 0.5
 * (the default), so s_k = max|X_k|^0.5 / max|W_k|^0.5 = sqrt(max|X_k| /
 * max|W_k|), formed in IEEE binary32 (a division and a square root, both
 * correctly rounded), clamped to [2^-14, 2^14] and rounded to FP16; s_k = 1
 * where either maximum is 0.  The smoothed operands are FP16: W' = fp16(W *
 * s) (the product of two FP16 values is exact, so it is rounded once) and
 * X' = fp16(X / s) with the quotient formed in IEEE binary32.
 * ------------------------------------------------------------------------- */
void orc_smooth_factors(const uint16_t* Xc, int Mc, const uint16_t* W, int N, int K,
                        uint16_t* s) {
    for (int k = 0; k < K; ++k) {
        float ax = 0.0f, aw = 0.0f;
        for (int m = 0; m < Mc; ++m) {
            float v = fabsf(orc_h2f(Xc[(size_t)m * K + k]));
            if (v > ax) ax = v;
        }
        for (int n = 0; n < N; ++n) {
            float v = fabsf(orc_h2f(W[(size_t)n * K + k]));
            if (v > aw) aw = v;
        }
        if (ax == 0.0f || aw == 0.0f) {
            s[k] = 0x3c00;                        /* 1.0 */
            continue;
        }
        float r = sqrtf(ax / aw);
        if (r < 0x1p-14f) r = 0x1p-14f;
        if (r > 0x1p14f) r = 0x1p14f;
        s[k] = orc_f2h(r);
    }
}

void orc_smooth_weights(const uint16_t* W, const uint16_t* s, int N, int K, uint16_t* Wp) {
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            Wp[(size_t)n * K + k] = orc_d2h(orc_h2d(W[(size_t)n * K + k]) * orc_h2d(s[k]));
}

void orc_smooth_act(const uint16_t* X, const uint16_t* s, int M, int K, uint16_t* Xp) {
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k)
            Xp[(size_t)m * K + k] = orc_f2h(orc_h2f(X[(size_t)m * K + k]) / orc_h2f(s[k]));
}

/* ---------------------------------------------------------------------------
 * The output-side step the gate_up GEMM's epilogue takes over ("Part5
 * LLM部署技术", 3. 实践扩展：QServe（W4A8KV4）, kernel fusion): the MLP of the
 * served models (Llama-3-8B, Qwen1.5-72B) applies SiLU to the gate half of
 * the fused gate_up projection and multiplies by the up half; the pages name
 * the models, not the formula, so this is the reading taken.  G and U are
 * the FP16 outputs of the two halves (M x I); H = fp16(silu(g) * u) with
 * silu(x) = x / (1 + exp(-x)), formed in binary64.  H is then quantized per
 * token (orc_quant_act) for the down projection.
 * ------------------------------------------------------------------------- */
void orc_silu_mul(const uint16_t* G, const uint16_t* U, long count, uint16_t* H) {
    for (long i = 0; i < count; ++i) {
        double g = orc_h2d(G[i]);
        double silu = g / (1.0 + exp(-g));
        H[i] = orc_d2h(silu * orc_h2d(U[i]));
    }
}

/* ---------------------------------------------------------------------------
 * 4-bit KV cache and decode attention over it ("QServe: Cuantificación
 * W4A8KV4 y Co-diseño del Sistema ...", abstract: 4-bit KV cache; "QServe:
 * W4A8KV4 Quantization and System Co-design ..." (velog notes), Insight:
 * the fused attention is made memory-bound so that KV4 pays off).  The pages
 * fix no format for the cache; the readings taken:
 *  - every (token, KV head) vector x of d FP16 values is quantized on its
 *    own, asymmetrically, to UINT4 codes with an FP16 scale s and an FP16
 *    offset m (the vector's minimum): x^ = s * q + m;
 *  - s = fp16(fl32(fl32(max - min) / 15)) and q = clamp(rne(fl32(fl32(x -
 *    min) / s)), 0, 15), each operation in IEEE binary32 (the kernel's
 *    precision, so that both sides take every integer decision alike); a
 *    vector whose s is 0 (constant, or a range below the FP16 resolution)
 *    gets q = 0 everywhere, so x^ = m;
 *  - decode attention: one query token per sequence; query head h reads KV
 *    head h / (Hq / Hkv) (grouped-query attention, as in the served
 *    Llama-3-8B); score_t = (q . k^_t) / sqrt(d) over the sequence's first
 *    L_b tokens; p = softmax(score); out = sum_t p_t v^_t, formed in binary64
 *    and rounded to FP16 once; a sequence of length 0 gives out = 0.
 * ------------------------------------------------------------------------- */
void orc_kv4_quant(const uint16_t* X, long rows, int d, uint8_t* q, uint16_t* s, uint16_t* m) {
    for (long r = 0; r < rows; ++r) {
        const uint16_t* x = X + r * d;
        float mn = orc_h2f(x[0]), mx = mn;
        uint16_t mn_bits = x[0];
        for (int i = 1; i < d; ++i) {
            float v = orc_h2f(x[i]);
            if (v < mn) { mn = v; mn_bits = x[i]; }
            if (v > mx) mx = v;
        }
        float range = mx - mn;
        uint16_t sh = orc_f2h(range / 15.0f);
        float sv = orc_h2f(sh);
        s[r] = sh;
        m[r] = (mn == 0.0f) ? 0 : mn_bits;   /* -0 and +0 are the same offset */
        for (int i = 0; i < d; ++i) {
            int c = 0;
            if (sv > 0.0f) {
                float t = (orc_h2f(x[i]) - mn) / sv;
                c = clampi((int)rne_f(t), 0, 15);
            }
            q[r * d + i] = (uint8_t)c;
        }
    }
}

/* x^ = s * q + m, exactly (binary64). */
void orc_kv4_dequant(const uint8_t* q, const uint16_t* s, const uint16_t* m, long rows, int d,
                     double* out) {
    for (long r = 0; r < rows; ++r) {
        double sv = orc_h2d(s[r]), mv = orc_h2d(m[r]);
        for (int i = 0; i < d; ++i) out[r * d + i] = sv * (double)q[r * d + i] + mv;
    }
}

/* Q: [B][Hq][d] FP16.  Codes qk, qv: [B][Hkv][L][d], one code per byte;
 * sk, mk, sv, mv: [B][Hkv][L] FP16; seqlen[b] <= L.  out: [B][Hq][d] FP16,
 * out64 (optional): the same before the FP16 rounding. */
void orc_kv4_decode_attention(const uint16_t* Q, const uint8_t* qk, const uint16_t* sk,
                              const uint16_t* mk, const uint8_t* qv, const uint16_t* sv,
                              const uint16_t* mv, const int* seqlen, int B, int Hq, int Hkv,
                              int L, int d, uint16_t* out, double* out64) {
    const int g = Hq / Hkv;
    double* score = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
    double* kh = (double*)malloc(sizeof(double) * d);
    for (int b = 0; b < B; ++b) {
        const int Lb = seqlen[b];
        for (int h = 0; h < Hq; ++h) {
            const int hk = h / g;
            const long base = ((long)b * Hkv + hk) * L;      /* first token row of (b, hk) */
            const uint16_t* qh = Q + ((long)b * Hq + h) * d;
            double* o64 = out64 ? out64 + ((long)b * Hq + h) * d : NULL;
            uint16_t* o = out + ((long)b * Hq + h) * d;
            if (Lb <= 0) {
                for (int i = 0; i < d; ++i) {
                    o[i] = 0;
                    if (o64) o64[i] = 0.0;
                }
                continue;
            }
            double mx = -INFINITY;
            for (int t = 0; t < Lb; ++t) {
                orc_kv4_dequant(qk + (base + t) * d, sk + base + t, mk + base + t, 1, d, kh);
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += orc_h2d(qh[i]) * kh[i];
                score[t] = acc / sqrt((double)d);
                if (score[t] > mx) mx = score[t];
            }
            double sum = 0.0;
            for (int t = 0; t < Lb; ++t) {
                score[t] = exp(score[t] - mx);
                sum += score[t];
            }
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int t = 0; t < Lb; ++t) {
                    const long r = base + t;
                    acc += score[t] * (orc_h2d(sv[r]) * (double)qv[r * d + i] + orc_h2d(mv[r]));
                }
                acc /= sum;
                if (o64) o64[i] = acc;
                o[i] = orc_d2h(acc);
            }
        }
    }
    free(score);
    free(kh);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
