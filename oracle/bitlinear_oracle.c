/*
 * bitlinear_oracle.c -- plain, slow, obviously-correct CPU oracle of the
 * inference-time BitLinear forward of BitNet b1.58 (W1.58A8).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with
 * the CUDA library; the two are written independently from the same pages.
 *
 * Sources (web pages; cited by title and section):
 *   [QG]  "BitNet" -- transformers quantization guide (Portuguese edition):
 *         numbered steps 1-3 of the quantisation recipe.
 *   [BG]  "Transformers 实战 BitNet 1.58 位量化：BitLinear 原理、量化流程与推理加载全指南"
 *         (2kiu.com walkthrough): section "BitLinear 的三步量化" (steps 1-3:
 *         absmean weight scale, ternary rounding, per-token absmax int8) and
 *         section "推理侧 BitLinear：打包权重、解包与缩放" (pack_weights,
 *         unpack_weights, BitLinear.forward order, input_scale*weight_scale
 *         rescale, sub-norm before quantising).
 *   [MD]  "BitNet" -- transformers model doc (Chinese / Portuguese editions):
 *         "模型详情" / model details (W1.58A8, absmean / per-token absmax,
 *         ReLU^2 FFN, subln) and BitNetConfig (hidden 2560, intermediate 6912,
 *         30 layers, rms_norm_eps 1e-5).
 *
 * Arithmetic conventions (readings where the pages are silent):
 *   - every scalar op is an IEEE binary32 op rounded to nearest-even (RN32)
 *     unless written as binary64 (RN64); build with -ffp-contract=off so no
 *     multiply-add is ever fused;
 *   - "round" is round-half-to-even (rintf under the default rounding mode);
 *   - sums that the pages write as mean()/pow(2).mean() are taken EXACTLY and
 *     rounded once to binary64 (ref_exact_sum_f64 below);
 *   - bf16 values travel as their uint16 bit patterns.
 *
 * Build:  gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 *         -o liboracle.so bitlinear_oracle.c -lm      (see oracle/build.py)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must be built without fast-math"
#endif

/* ------------------------------------------------------------------------ */
/* Exact summation of binary64 values (superaccumulator).                   */
/*                                                                          */
/* Every finite double is an integer multiple of 2^-1074.  We keep the sum  */
/* as a big integer in base 2^32 "digits" (digit i weighs 2^(32 i - 1074)), */
/* add each value's 53-bit significand at its bit position, and round the   */
/* final integer to the nearest double, ties to even.  The result is the    */
/* correctly rounded exact sum, the same quantity Python's math.fsum        */
/* returns, which the tests use as an independent check.                    */
/* ------------------------------------------------------------------------ */
#define SA_NDIG 72 /* 72*32 = 2304 bits > 2098 needed + carry headroom */

typedef struct {
    int64_t d[SA_NDIG];
    int64_t pending; /* additions since the last carry normalisation */
} superacc;

static void sa_init(superacc* a) { memset(a, 0, sizeof(*a)); }

/* Propagate carries so that digits 0..SA_NDIG-2 lie in [0, 2^32). */
static void sa_normalize(superacc* a) {
    for (int i = 0; i < SA_NDIG - 1; ++i) {
        int64_t carry = a->d[i] >> 32; /* floor division (gcc: arithmetic shift) */
        a->d[i] -= carry * (int64_t)4294967296LL;
        a->d[i + 1] += carry;
    }
    a->pending = 0;
}

static void sa_add(superacc* a, double v) {
    if (v == 0.0) return;
    uint64_t bits;
    memcpy(&bits, &v, sizeof bits);
    int negative = (int)(bits >> 63);
    int biased = (int)((bits >> 52) & 0x7FF);
    uint64_t sig = bits & 0xFFFFFFFFFFFFFull;
    int pos; /* bit position of sig's lowest bit, counted from 2^-1074 */
    if (biased == 0) {
        pos = 0; /* subnormal: value = sig * 2^-1074 */
    } else {
        sig |= (uint64_t)1 << 52; /* value = sig * 2^(biased-1075) */
        pos = biased - 1;
    }
    int j = pos >> 5, s = pos & 31;
    unsigned __int128 w = (unsigned __int128)sig << s; /* at most 84 bits */
    int64_t c0 = (int64_t)(uint32_t)w;
    int64_t c1 = (int64_t)(uint32_t)(w >> 32);
    int64_t c2 = (int64_t)(uint32_t)(w >> 64);
    if (negative) {
        a->d[j] -= c0; a->d[j + 1] -= c1; a->d[j + 2] -= c2;
    } else {
        a->d[j] += c0; a->d[j + 1] += c1; a->d[j + 2] += c2;
    }
    if (++a->pending >= ((int64_t)1 << 30)) sa_normalize(a);
}

/* bit b (counted from 2^-1074) of a normalised, non-negative accumulator */
static int sa_bit(const superacc* a, int b) {
    return (int)((a->d[b >> 5] >> (b & 31)) & 1);
}

/* any bit set strictly below position b? */
static int sa_any_below(const superacc* a, int b) {
    int j = b >> 5, s = b & 31;
    for (int i = 0; i < j; ++i)
        if (a->d[i]) return 1;
    if (s && (a->d[j] & (((int64_t)1 << s) - 1))) return 1;
    return 0;
}

static double sa_round(superacc* a) {
    sa_normalize(a);
    int negative = a->d[SA_NDIG - 1] < 0;
    if (negative) {
        for (int i = 0; i < SA_NDIG; ++i) a->d[i] = -a->d[i];
        sa_normalize(a);
    }
    int top = -1;
    for (int i = SA_NDIG - 1; i >= 0; --i)
        if (a->d[i]) { top = i; break; }
    if (top < 0) return 0.0;
    int hb = 32 * top + (63 - __builtin_clzll((uint64_t)a->d[top])); /* highest set bit */
    double r;
    if (hb < 53) {
        uint64_t m = (uint64_t)a->d[0] | ((uint64_t)a->d[1] << 32); /* exact, < 2^53 */
        r = ldexp((double)m, -1074);
    } else {
        uint64_t m = 0;
        for (int b = hb; b >= hb - 52; --b) m = (m << 1) | (uint64_t)sa_bit(a, b);
        int round_bit = sa_bit(a, hb - 53);
        int sticky = sa_any_below(a, hb - 53);
        int e = hb - 52 - 1074;
        if (round_bit && (sticky || (m & 1))) {
            m += 1;
            if (m == ((uint64_t)1 << 53)) { m >>= 1; e += 1; }
        }
        r = ldexp((double)m, e); /* overflow gives inf, as IEEE rounding would */
    }
    return negative ? -r : r;
}

/* Correctly rounded binary64 value of the exact sum v[0] + ... + v[n-1]. */
double ref_exact_sum_f64(const double* v, int64_t n) {
    superacc a;
    sa_init(&a);
    for (int64_t i = 0; i < n; ++i) sa_add(&a, v[i]);
    return sa_round(&a);
}

/* ------------------------------------------------------------------------ */
/* bf16 <-> binary32                                                        */
/* ------------------------------------------------------------------------ */
float ref_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of a binary32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even; NaN stays NaN. */
uint16_t ref_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) /* NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;          /* truncated result */
    uint32_t rest = u & 0xFFFFu;      /* discarded low half */
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1; /* may carry into exponent: correct */
    return (uint16_t)keep;
}

/* ------------------------------------------------------------------------ */
/* Weight side: absmean scale, ternary codes, 2-bit packing.               */
/* ------------------------------------------------------------------------ */

/* [BG] "BitLinear 的三步量化" step 1 / [QG] step 1: the per-tensor scale is the
 * mean of |W| over the whole matrix, clamped below at 1e-5.  Returned as beta
 * (the absmean itself); the multiplier used for rounding is 1/beta.
 *   beta = max( RN32( RN64(sum|W|) / (double)(N*K) ), 1e-5f )                */
float ref_weight_scale(const float* W, int64_t N, int64_t K) {
    superacc a;
    sa_init(&a);
    int64_t n = N * K;
    for (int64_t i = 0; i < n; ++i) sa_add(&a, fabs((double)W[i]));
    double s = sa_round(&a);
    double mean = s / (double)n;
    float beta = (float)mean;
    const float floor_ = 1e-5f;
    return beta < floor_ ? floor_ : beta;
}

/* [BG] step 2 / [QG] step 2: t = clamp(round(W * s_w), -1, 1), s_w = 1/beta. */
void ref_ternarize(const float* W, int64_t n, float beta, int8_t* t) {
    float s_w = 1.0f / beta;
    for (int64_t i = 0; i < n; ++i) {
        float p = W[i] * s_w;
        float r = rintf(p);
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        t[i] = (int8_t)r;
    }
}

/* [BG] "推理侧 BitLinear" pack_weights: each ternary value is stored as t+1 in
 * two bits, four per byte, the packed matrix having a quarter of the rows.
 * Byte P[r,k] holds, in its bit pair i (bits 2i..2i+1), the code of row
 * i*(N/4) + r of column k ("block" layout: bit pair i is the i-th quarter of
 * the rows).  Returns 0, or -1 if N is not a multiple of 4 or a value is not
 * in {-1,0,1}.                                                             */
int ref_pack(const int8_t* t, int64_t N, int64_t K, uint8_t* P) {
    if (N % 4 != 0) return -1;
    int64_t R = N / 4;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = 0;
            for (int i = 0; i < 4; ++i) {
                int v = t[(i * R + r) * K + k];
                if (v < -1 || v > 1) return -1;
                byte |= (unsigned)(v + 1) << (2 * i);
            }
            P[r * K + k] = (uint8_t)byte;
        }
    }
    return 0;
}

/* [BG] "推理侧 BitLinear" unpack_weights: bit pair i selected by the mask
 * 3 << 2i, shifted down, minus one.  (A bit pair 11, which pack never
 * writes, decodes arithmetically to +2.)                                   */
void ref_unpack(const uint8_t* P, int64_t N, int64_t K, int8_t* t) {
    int64_t R = N / 4;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = P[r * K + k];
            for (int i = 0; i < 4; ++i) {
                unsigned mask = 3u << (2 * i);
                int code = (int)((byte & mask) >> (2 * i));
                t[(i * R + r) * K + k] = (int8_t)(code - 1);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Activation side: optional RMSNorm, per-token absmax int8 quantisation.   */
/* ------------------------------------------------------------------------ */

/* Plain bf16 -> binary32 widening of a whole buffer (the no-norm path). */
void ref_bf16_to_f32_buf(const uint16_t* x, int64_t n, float* h) {
    for (int64_t i = 0; i < n; ++i) h[i] = ref_bf16_to_f32(x[i]);
}

/* RMSNorm applied by BitLinear.forward before quantising ([BG] "推理侧 BitLinear",
 * forward order; eps = rms_norm_eps = 1e-5 in [MD] BitNetConfig).  The pages
 * give no formula; this is the standard root-mean-square norm:
 *   SS = RN64( sum_k x_k^2 )           (exact sum; bf16^2 is exact in binary64)
 *   r  = RN32( 1 / sqrt( SS/K + eps ) ) with each of /, +, sqrt, / in binary64
 *   h_k = RN32( RN32(x_k * r) * g_k )   (gain applied after the rms factor)
 * x, g are bf16 bit patterns; g may be NULL (unit gain: h_k = RN32(x_k * r)). */
void ref_rmsnorm(const uint16_t* x, const uint16_t* g, float eps, int64_t M, int64_t K,
                 float* h, float* r_out) {
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xr = x + m * K;
        superacc a;
        sa_init(&a);
        for (int64_t k = 0; k < K; ++k) {
            double xv = (double)ref_bf16_to_f32(xr[k]);
            sa_add(&a, xv * xv); /* exact: 8-bit significand squared */
        }
        double ss = sa_round(&a);
        double ms = ss / (double)K;
        double v = ms + (double)eps;
        double sd = sqrt(v);
        double rd = 1.0 / sd;
        float r = (float)rd;
        if (r_out) r_out[m] = r;
        for (int64_t k = 0; k < K; ++k) {
            float xv = ref_bf16_to_f32(xr[k]);
            float u = xv * r;
            h[m * K + k] = g ? u * ref_bf16_to_f32(g[k]) : u;
        }
    }
}

/* [BG] "BitLinear 的三步量化" step 3 / [QG] step 3: per token (per row, the
 * reduction runs over the last dimension) absmax scaling to int8:
 *   s_x = RN32( 127 / max(max_k |h_k|, 1e-5) )
 *   q_k = clamp( round(RN32(h_k * s_x)), -128, 127 )
 * rowsum[m] = sum_k q[m,k] is also returned (an exact integer).           */
void ref_act_quant(const float* h, int64_t M, int64_t K, int8_t* q, float* s_x,
                   int32_t* rowsum) {
    for (int64_t m = 0; m < M; ++m) {
        const float* hr = h + m * K;
        float mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(hr[k]);
            if (a > mx) mx = a;
        }
        const float floor_ = 1e-5f;
        if (mx < floor_) mx = floor_;
        float s = 127.0f / mx;
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float p = hr[k] * s;
            float r = rintf(p);
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            q[m * K + k] = (int8_t)r;
            sum += (int32_t)r;
        }
        s_x[m] = s;
        if (rowsum) rowsum[m] = sum;
    }
}

/* ------------------------------------------------------------------------ */
/* Matmul and rescale.                                                      */
/* ------------------------------------------------------------------------ */

/* [BG] "推理侧 BitLinear": F.linear of the int8 activations with the unpacked
 * ternary weights, accumulated exactly in int32:
 *   acc[m,n] = sum_k q[m,k] * t[n,k]                                       */
void ref_ternary_matmul(const int8_t* q, const int8_t* t, int64_t M, int64_t K, int64_t N,
                        int32_t* acc) {
    for (int64_t m = 0; m < M; ++m) {
        const int8_t* qr = q + m * K;
        /* the outputs of a row are independent exact integer sums: the
         * OpenMP build (liboracle_omp.so) computes them on all host cores,
         * the plain build one after another, with identical results */
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* tr = t + n * K;
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int32_t)qr[k] * (int32_t)tr[k];
            acc[m * N + n] = s;
        }
    }
}

/* [BG] "推理侧 BitLinear" post_quant_process: undo both scales.  With beta the
 * absmean (weight scale) and s_x the activation multiplier:
 *   y[m,n] = RN32( RN32(acc[m,n] * beta) / s_x[m] )                        */
void ref_rescale(const int32_t* acc, const float* s_x, float beta, int64_t M, int64_t N,
                 float* y) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float a = (float)acc[m * N + n]; /* exact: |acc| < 2^24 */
            float u = a * beta;
            y[m * N + n] = u / s_x[m];
        }
    }
}

void ref_f32_to_bf16_buf(const float* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = ref_f32_to_bf16(y[i]);
}

/* Whole BitLinear forward ([BG] "推理侧 BitLinear", in its order: optional
 * RMSNorm, unpack, activation quant, matmul, rescale).  x bf16 [M,K]; gain
 * bf16 [K] or NULL for no norm; P packed [N/4,K]; y fp32 [M,N].  Optional
 * outputs q [M,K], s_x [M], acc [M,N] may be NULL.  Returns 0, or -1 on a
 * bad shape or allocation failure.                                         */
int ref_forward(const uint16_t* x, const uint16_t* gain, int use_norm, float eps,
                const uint8_t* P, float beta, int64_t M, int64_t K, int64_t N, float* y,
                int8_t* q_out, float* sx_out, int32_t* acc_out) {
    if (M < 0 || K <= 0 || N <= 0 || N % 4 != 0) return -1;
    float* h = (float*)malloc(sizeof(float) * (size_t)(M * K + 1));
    int8_t* q = (int8_t*)malloc((size_t)(M * K + 1));
    float* sx = (float*)malloc(sizeof(float) * (size_t)(M + 1));
    int8_t* t = (int8_t*)malloc((size_t)(N * K));
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * N + 1));
    int rc = -1;
    if (!h || !q || !sx || !t || !acc) goto done;
    if (use_norm)
        ref_rmsnorm(x, gain, eps, M, K, h, NULL);
    else
        ref_bf16_to_f32_buf(x, M * K, h);
    ref_unpack(P, N, K, t);
    ref_act_quant(h, M, K, q, sx, NULL);
    ref_ternary_matmul(q, t, M, K, N, acc);
    ref_rescale(acc, sx, beta, M, N, y);
    if (q_out) memcpy(q_out, q, (size_t)(M * K));
    if (sx_out) memcpy(sx_out, sx, sizeof(float) * (size_t)M);
    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));
    rc = 0;
done:
    free(h); free(q); free(sx); free(t); free(acc);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* FFN block glue ([MD] model details: ReLU^2 FFN, subln; [BG] "推理侧 BitLinear":
 * ffn_sub_norm normalises the MLP activation before it is quantised).      */
/* ------------------------------------------------------------------------ */

/* z = bf16( RN32( RN32(relu(a) * relu(a)) * b ) ), a = gate, b = up (bf16). */
void ref_relu2_mul(const uint16_t* a, const uint16_t* b, int64_t n, uint16_t* z) {
    for (int64_t i = 0; i < n; ++i) {
        float av = ref_bf16_to_f32(a[i]);
        float ra = av > 0.0f ? av : 0.0f;
        float sq = ra * ra;
        float v = sq * ref_bf16_to_f32(b[i]);
        z[i] = ref_f32_to_bf16(v);
    }
}

/* out = bf16( x + d ), all bf16. */
void ref_residual_add(const uint16_t* x, const uint16_t* d, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i)
        out[i] = ref_f32_to_bf16(ref_bf16_to_f32(x[i]) + ref_bf16_to_f32(d[i]));
}

/* One FFN block at M tokens, hidden H, intermediate I:
 *   hq      = quant( RMSNorm(x, g_in) )
 *   a, b    = bf16( BitLinear_gate(hq) ), bf16( BitLinear_up(hq) )
 *   z       = relu(a)^2 * b
 *   d       = bf16( BitLinear_down( quant( RMSNorm(z, g_sub) ) ) )
 *   x_out   = bf16( x + d )
 * P_gate, P_up: [I/4, H]; P_down: [H/4, I].  x_out may alias x.           */
int ref_ffn_block(const uint16_t* x, const uint16_t* g_in, const uint16_t* g_sub, float eps,
                  const uint8_t* P_gate, float beta_gate, const uint8_t* P_up, float beta_up,
                  const uint8_t* P_down, float beta_down, int64_t M, int64_t H, int64_t I,
                  uint16_t* x_out) {
    int rc = -1;
    float* yf = (float*)malloc(sizeof(float) * (size_t)(M * (I > H ? I : H) + 1));
    uint16_t* a = (uint16_t*)malloc(2 * (size_t)(M * I + 1));
    uint16_t* b = (uint16_t*)malloc(2 * (size_t)(M * I + 1));
    uint16_t* z = (uint16_t*)malloc(2 * (size_t)(M * I + 1));
    uint16_t* d = (uint16_t*)malloc(2 * (size_t)(M * H + 1));
    if (!yf || !a || !b || !z || !d) goto done;
    if (ref_forward(x, g_in, 1, eps, P_gate, beta_gate, M, H, I, yf, NULL, NULL, NULL)) goto done;
    ref_f32_to_bf16_buf(yf, M * I, a);
    if (ref_forward(x, g_in, 1, eps, P_up, beta_up, M, H, I, yf, NULL, NULL, NULL)) goto done;
    ref_f32_to_bf16_buf(yf, M * I, b);
    ref_relu2_mul(a, b, M * I, z);
    if (ref_forward(z, g_sub, 1, eps, P_down, beta_down, M, I, H, yf, NULL, NULL, NULL)) goto done;
    ref_f32_to_bf16_buf(yf, M * H, d);
    ref_residual_add(x, d, M * H, x_out);
    rc = 0;
done:
    free(yf); free(a); free(b); free(z); free(d);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Online quantisation-aware training.  "Transformers 实战 BitNet 1.58 位量化"
 * walkthrough: "量化器参数：BitNetQuantConfig 详解" (AutoBitLinear with
 * quantization_mode "online" quantises the weights on every forward through
 * WeightQuant) and "BitLinear 的三步量化" (steps 1-3, and the straight-through
 * estimator of both quantisers' backward).                                 */
/* ------------------------------------------------------------------------ */

/* The online forward: the weight scale and the ternary weights are derived
 * from the fp32 master weights W [N,K] on this call (steps 1-2), then the
 * forward is the BitLinear forward of ref_forward on them.  beta_out (the
 * absmean) and t_out [N,K] are optional outputs.  Returns 0, or -1 on a bad
 * shape or allocation failure.                                             */
int ref_online_forward(const uint16_t* x, const uint16_t* gain, int use_norm, float eps,
                       const float* W, int64_t M, int64_t K, int64_t N, float* y,
                       float* beta_out, int8_t* t_out) {
    if (M < 0 || K <= 0 || N <= 0 || N % 4 != 0) return -1;
    int8_t* t = (int8_t*)malloc((size_t)(N * K));
    uint8_t* P = (uint8_t*)malloc((size_t)(N / 4 * K));
    int rc = -1;
    if (!t || !P) goto done;
    float beta = ref_weight_scale(W, N, K);
    ref_ternarize(W, N * K, beta, t);
    if (ref_pack(t, N, K, P)) goto done;
    if (ref_forward(x, gain, use_norm, eps, P, beta, M, K, N, y, NULL, NULL, NULL)) goto done;
    if (beta_out) *beta_out = beta;
    if (t_out) memcpy(t_out, t, (size_t)(N * K));
    rc = 0;
done:
    free(t); free(P);
    return rc;
}

/* The backward of the layer under the straight-through estimator: both
 * quantisers pass the gradient through unchanged (grad_input = grad_output),
 * so the gradients are those of the linear layer on the dequantised operands
 * the forward multiplied (step 2: weight = round-and-clamp(W * scale) / scale;
 * step 3: activation = round-and-clamp(x * scale) / scale):
 *   W_q[n,k] = RN32( t[n,k] / s_w ),  s_w = RN32(1 / beta)
 *   x_q[m,k] = RN32( q[m,k] / s_x[m] )
 *   gx[m,k]  = sum_n gy[m,n] * W_q[n,k]      (grad of the input)
 *   gw[n,k]  = sum_m gy[m,n] * x_q[m,k]      (grad of the master weight)
 * gy [M,N] binary32; the products of two binary32 values are exact in
 * binary64 and the sums are taken in binary64 in index order.              */
void ref_ste_backward(const float* gy, const int8_t* q, const float* s_x, const int8_t* t,
                      float beta, int64_t M, int64_t K, int64_t N, double* gx, double* gw) {
    float s_w = 1.0f / beta;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                float wq = (float)t[n * K + k] / s_w;
                s += (double)gy[m * N + n] * (double)wq;
            }
            gx[m * K + k] = s;
        }
    }
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                float xq = (float)q[m * K + k] / s_x[m];
                s += (double)gy[m * N + n] * (double)xq;
            }
            gw[n * K + k] = s;
        }
    }
}
