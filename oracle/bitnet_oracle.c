/*
 * bitnet_oracle.c -- CPU oracle for the BitLinear / H-BitLinear forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or calls this
 * file; only the test-suite, the smoke check and the timed CPU baseline in bench.py do.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * It states the method as plainly as possible: plain loops, double precision wherever the
 * pages do not fix a precision, int64 accumulation, no blocking or fusion.  Where a floating
 * point value decides an integer (a ternary weight, an activation code), the decision is
 * taken in IEEE fp32, the precision the CUDA kernels use, so that both sides round the same
 * way; every such place says so.  OpenMP only splits independent token / weight rows
 * between host cores.
 *
 * Sources (page title, section):
 *   [b1.58]   "The Era of 1-bit LLMs: All Large Language Models are in 1.58 Bits" -- summary
 *             page (gptget.net/papers/2402.17764), sections 方法论 and 方法详解: weights are
 *             constrained to {-1,0,+1} with an absmean quantisation function; BitLinear
 *             replaces nn.Linear.
 *   [2B4T]    BitNet b1.58 2B4T article (itdecent.cn/p/6fce9dbc5e50), section 一.1 (ternary
 *             weights, five trits in one byte: 2,0,1,2,1 -> 178, 99.06 % of optimum) and
 *             section 一.2 (BitLinear: absmean weights, absmax 8-bit activations, W1.58A8;
 *             multiplying by 1 adds, by -1 subtracts, by 0 skips).
 *   [v2]      BitNet v2 write-up (kaiyunao.com), paragraphs on H-BitLinear: an online
 *             Hadamard transform (entries +-1, mutually orthogonal rows) is applied to the
 *             activations before they are quantised; 8-bit and 4-bit activation variants.
 *   [v2-abs]  "BitNet v2: Native 4-bit Activations with Hadamard Transformation for 1-bit
 *             LLMs", abstract (chatpaper.ai).
 *
 * Readings taken where the pages print no formula (each is listed in the design notes):
 *   gamma = fp32(max(mean|W|, 1e-5)) with the mean in double; q = clip(rint(w / gamma), -1, 1)
 *   with an fp32 IEEE division and round-half-even; Hadamard = Sylvester order, scaled by
 *   1/sqrt(K) (orthonormal), size K; output = bf16_rn(acc * d * gamma).
 *   Activation quantisers: the [v2] write-up says INT8 and INT4 "respectively" take their own
 *   strategy, and names absmax for the 4-bit activations of the post-training baselines only;
 *   the pages name two quantisation functions, absmax (8-bit activations, [2B4T] 一.2) and
 *   absmean ([b1.58]).  So INT8 = per-token absmax, Q = 127, eps 1e-5, round-half-even, clip to
 *   [-128, 127], d = max|z| / 127; INT4 = per-token absmean, the mean |z| of a token mapped to
 *   code sqrt(7), eps 1e-5, clip to [-8, 7], d = mean|z| / sqrt(7).  Variant INT4 quantiser
 *   (not the default): absmax with Q = 7.  Low-bit Q / K / V states ([v2] Tables 2-3 vary
 *   their width): the absmax rule per token or per head with Q = 2^(bits-1) - 1, stored as a
 *   little-endian bit stream of two's complement fields.
 *   Variant weight + activation rotation (not the default): the rows of W are transformed by
 *   the same orthonormal Hadamard before the absmean ternarisation, W' = W H / sqrt(K), so that
 *   W' (H x / sqrt(K)) = W x; the rotated rows are rounded to fp32 once, then ternarised.
 *
 * Parity pins live in tests/test_oracle_pins.py: every exported function is checked there
 * against something independent of it (a page's worked example, a closed form, a library
 * routine, brute force).  The pins fix the arithmetic of the readings above; the readings
 * themselves (eps, rounding, the INT4 rule, the 1/sqrt(K) scale) are not printed on the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------------- */
/* bf16 <-> double                                                                         */
/* ------------------------------------------------------------------------------------- */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double straight to bf16 (8 significant bits), ties to even, without passing
 * through binary32 (which would round twice). */
static uint16_t double_to_bf16_rn(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isnan(v)) return 0x7FC0u;
    if (a == 0.0) return sign;
    int e;
    double f = frexp(a, &e);           /* a = f * 2^e, 0.5 <= f < 1 */
    int unbiased = e - 1;              /* a = 1.xxx * 2^unbiased */
    if (unbiased < -126) {             /* subnormal range: fixed quantum 2^-133 */
        double r = nearbyint(ldexp(a, 133));
        return (uint16_t)(sign | (uint16_t)r);   /* r == 128 is the smallest normal: still right */
    }
    double r = nearbyint(f * 256.0);   /* 8 significant bits, round half to even */
    if (r >= 256.0) { r = 128.0; unbiased += 1; }
    if (unbiased > 127) return (uint16_t)(sign | 0x7F80u);  /* overflow to inf */
    uint16_t exp_field = (uint16_t)(unbiased + 127);
    uint16_t mant = (uint16_t)((int)r - 128);
    return (uint16_t)(sign | (exp_field << 7) | mant);
}

uint16_t oracle_double_to_bf16(double v) { return double_to_bf16_rn(v); }
double oracle_bf16_to_double(uint16_t h) { return bf16_to_double(h); }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------- */
/* Step 1: absmean ternarisation of the weights  [b1.58 方法论/方法详解], [2B4T 一.2]       */
/* ------------------------------------------------------------------------------------- */

/* Sum of |w| over all weights, in double, in index order. */
double oracle_abs_sum_bf16(const uint16_t *w, int64_t n) {
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += fabs(bf16_to_double(w[i]));
    return s;
}

/* gamma = mean |W| over the whole tensor (one scale per tensor), guarded away from zero. */
float oracle_absmean_gamma(const uint16_t *w, int64_t n) {
    double mean = oracle_abs_sum_bf16(w, n) / (double)n;
    if (mean < 1e-5) mean = 1e-5;
    return (float)mean;
}

/* q = RoundClip(w / gamma, -1, 1).  The division and the rounding decide an integer, so they
 * are done in IEEE fp32 (the kernel's precision): one correctly rounded division, then
 * round-half-to-even (nearbyintf under the default rounding mode). */
void oracle_ternarize(const uint16_t *w, int64_t n, float gamma, int8_t *q) {
    for (int64_t i = 0; i < n; ++i) {
        float wf = (float)bf16_to_double(w[i]);
        volatile float r = wf / gamma;          /* volatile: keep it one fp32 division */
        float t = nearbyintf(r);
        if (t > 1.0f) t = 1.0f;
        if (t < -1.0f) t = -1.0f;
        q[i] = (int8_t)t;
    }
}

/* The same absmean ternarisation on fp32 weights: the Hadamard-rotated rows W' = W H / sqrt(K)
 * of the weight + activation rotation [v2: Hadamard rotation of the weights and the activations,
 * or of the activations only].  gamma = fp32(max(mean |w'|, 1e-5)), the sum in double; then
 * q = RoundClip(w' / gamma, -1, 1) with one IEEE fp32 division and round-half-to-even. */
float oracle_absmean_gamma_f32(const float *w, int64_t n) {
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += fabs((double)w[i]);
    double mean = s / (double)n;
    if (mean < 1e-5) mean = 1e-5;
    return (float)mean;
}

void oracle_ternarize_f32(const float *w, int64_t n, float gamma, int8_t *q) {
    for (int64_t i = 0; i < n; ++i) {
        volatile float r = w[i] / gamma;
        float t = nearbyintf(r);
        if (t > 1.0f) t = 1.0f;
        if (t < -1.0f) t = -1.0f;
        q[i] = (int8_t)t;
    }
}

/* ------------------------------------------------------------------------------------- */
/* Weight storage                                                                          */
/* ------------------------------------------------------------------------------------- */

/* 2-bit storage of the ternary weights (the pages print no GPU layout; this is the layout the
 * library defines).  Row-major [N][K/16] little-endian 32-bit words.  Word g of row n holds
 * k = 16g .. 16g+15.  Each weight is stored as the offset code u = q + 1 in {0,1,2}; weight
 * k = 16g + 4p + j (p, j in 0..3) sits at bits 8j + 2p of the word. */
void oracle_pack_ternary(const int8_t *q, int64_t N, int64_t K, uint32_t *wp) {
    int64_t words = K / 16;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < words; ++g) {
            uint32_t word = 0;
            for (int p = 0; p < 4; ++p) {
                for (int j = 0; j < 4; ++j) {
                    int64_t k = 16 * g + 4 * p + j;
                    uint32_t u = (uint32_t)(q[n * K + k] + 1);
                    word |= u << (8 * j + 2 * p);
                }
            }
            wp[n * words + g] = word;
        }
    }
}

/* Inverse of oracle_pack_ternary.  Returns the number of fields holding the unused code 3. */
int64_t oracle_unpack_ternary(const uint32_t *wp, int64_t N, int64_t K, int8_t *q) {
    int64_t words = K / 16, bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < words; ++g) {
            uint32_t word = wp[n * words + g];
            for (int p = 0; p < 4; ++p) {
                for (int j = 0; j < 4; ++j) {
                    uint32_t u = (word >> (8 * j + 2 * p)) & 3u;
                    if (u == 3u) ++bad;
                    q[n * K + 16 * g + 4 * p + j] = (int8_t)((int)u - 1);
                }
            }
        }
    }
    return bad;
}

/* Base-3 storage, five trits per byte, first trit most significant  [2B4T 一.1]:
 * digits d0..d4 in {0,1,2} -> d0*81 + d1*27 + d2*9 + d3*3 + d4  (2,0,1,2,1 -> 178).
 * A ragged tail is padded with digit 0. */
void oracle_pack_base3(const uint8_t *digits, int64_t n, uint8_t *out) {
    int64_t nbytes = (n + 4) / 5;
    for (int64_t b = 0; b < nbytes; ++b) {
        unsigned v = 0;
        for (int i = 0; i < 5; ++i) {
            int64_t idx = 5 * b + i;
            unsigned d = idx < n ? digits[idx] : 0u;
            v = v * 3u + d;
        }
        out[b] = (uint8_t)v;
    }
}

void oracle_unpack_base3(const uint8_t *bytes, int64_t n, uint8_t *digits) {
    int64_t nbytes = (n + 4) / 5;
    for (int64_t b = 0; b < nbytes; ++b) {
        unsigned v = bytes[b];
        uint8_t d[5];
        for (int i = 4; i >= 0; --i) { d[i] = (uint8_t)(v % 3u); v /= 3u; }
        for (int i = 0; i < 5; ++i) {
            int64_t idx = 5 * b + i;
            if (idx < n) digits[idx] = d[i];
        }
    }
}

/* Base-3 storage of a ternary matrix for the decode product, built on oracle_pack_base3
 * [2B4T 一.1]: row n is ceil(K/20) 32-bit little-endian words; byte i of word w holds the offset
 * codes u = q + 1 of weights k = 20w + 5i .. 20w + 5i + 4 as one base-3 number, first weight
 * most significant; weights k >= K are stored as u = 1 (q = 0).  1.6 bits per weight. */
void oracle_pack_ternary_base3(const int8_t *q, int64_t N, int64_t K, uint32_t *out) {
    const int64_t words = (K + 19) / 20;
    uint8_t *dig = malloc((size_t)(words * 20));
    if (!dig) return;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < words * 20; ++k)
            dig[k] = k < K ? (uint8_t)(q[n * K + k] + 1) : 1u;
        oracle_pack_base3(dig, words * 20, (uint8_t *)(out + n * words));
    }
    free(dig);
}

/* Inverse of oracle_pack_ternary_base3.  Returns the number of bytes that are not valid base-3
 * numbers (>= 243) plus the number of padding weights not stored as u = 1. */
int64_t oracle_unpack_ternary_base3(const uint32_t *in, int64_t N, int64_t K, int8_t *q) {
    const int64_t words = (K + 19) / 20;
    uint8_t *dig = malloc((size_t)(words * 20));
    if (!dig) return -1;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *bytes = (const uint8_t *)(in + n * words);
        for (int64_t b = 0; b < words * 4; ++b) bad += bytes[b] >= 243;
        oracle_unpack_base3(bytes, words * 20, dig);
        for (int64_t k = 0; k < words * 20; ++k) {
            if (k < K) q[n * K + k] = (int8_t)((int)dig[k] - 1);
            else bad += dig[k] != 1;
        }
    }
    free(dig);
    return bad;
}

/* ------------------------------------------------------------------------------------- */
/* Before step 2: RMS normalisation of each token row  [2B4T 一.3: subln normalisation in  */
/* place of LayerNorm], [v2: LLaMA-like components with RMS normalisation]                 */
/* ------------------------------------------------------------------------------------- */

/* y = x * g / sqrt(mean_k(x_k^2) + eps) per row, in double; g is a bf16 gain per feature
 * (NULL: 1).  The pages name the normalisation only; this is the plainest reading of "RMS
 * normalisation", applied to the token row right before its quantisation (and before the
 * Hadamard transform in H-BitLinear). */
void oracle_rmsnorm(const double *x, int64_t M, int64_t K, const uint16_t *g, double eps,
                    double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const double *row = x + m * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += row[k] * row[k];
        const double r = 1.0 / sqrt(ss / (double)K + eps);
        for (int64_t k = 0; k < K; ++k)
            y[m * K + k] = row[k] * r * (g ? bf16_to_double(g[k]) : 1.0);
    }
}

/* ------------------------------------------------------------------------------------- */
/* Step 2: online Hadamard transform per token  [v2, H-BitLinear], [v2-abs]                */
/* ------------------------------------------------------------------------------------- */

/* z = (1/sqrt(K)) * H_K * x for every row, H_K in Sylvester order (H_2K = [[H,H],[H,-H]]),
 * computed by the in-place butterfly (fast Walsh-Hadamard transform) in double.  K must be a
 * power of two. */
void oracle_fwht(const double *x, int64_t M, int64_t K, double *z) {
    double scale = 1.0 / sqrt((double)K);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double *row = z + m * K;
        memcpy(row, x + m * K, (size_t)K * sizeof(double));
        for (int64_t h = 1; h < K; h *= 2) {
            for (int64_t i = 0; i < K; i += 2 * h) {
                for (int64_t j = i; j < i + h; ++j) {
                    double a = row[j], b = row[j + h];
                    row[j] = a + b;
                    row[j + h] = a - b;
                }
            }
        }
        for (int64_t j = 0; j < K; ++j) row[j] *= scale;
    }
}

/* ------------------------------------------------------------------------------------- */
/* Step 3: per-token activation quantisation: absmax (INT8) [2B4T 一.2], absmean (INT4) [v2]    */
/* ------------------------------------------------------------------------------------- */

/* Per-token absmax (INT8, and the INT4 variant).
 * For each row: m = max|z|, s = Q / max(m, 1e-5), c = clip(rint(z * s), -Q-1, Q), d = max(m, 1e-5) / Q,
 * with Q = 127 for 8-bit and Q = 7 for 4-bit codes.  The codes are decided in IEEE fp32 on
 * fp32 inputs (the kernel's precision).  If pre != NULL it receives z * s in double, the
 * unrounded value, so a test can see how close each code was to a rounding boundary.
 * rowsum (optional) receives the sum of the codes of each row. */
void oracle_quant_act(const float *z, int64_t M, int64_t K, int bits, int8_t *codes,
                      float *d, double *pre, int64_t *rowsum) {
    const float Q = bits == 4 ? 7.0f : 127.0f;
    const float lo = bits == 4 ? -8.0f : -128.0f;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const float *row = z + m * K;
        float mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(row[k]);
            if (a > mx) mx = a;
        }
        float g = mx < 1e-5f ? 1e-5f : mx;
        volatile float s = Q / g;
        volatile float dq = g / Q;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            volatile float v = row[k] * s;
            float t = nearbyintf(v);
            if (t > Q) t = Q;
            if (t < lo) t = lo;
            codes[m * K + k] = (int8_t)t;
            sum += (int64_t)t;
            if (pre) pre[m * K + k] = (double)row[k] * (double)Q / (double)g;
        }
        d[m] = dq;
        if (rowsum) rowsum[m] = sum;
    }
}

/*
 * INT4 quantiser with an absmean scale [v2: INT8 and INT4 each take their own strategy, whose
 * formulas are not printed; the pages' other quantisation function, the weights' absmean of
 * b1.58 / 2B4T 一.2, gives the form].  Reading: per token row, beta = mean |z| (in double, rounded to fp32 once), g = max(beta,
 * 1e-5); the mean magnitude is mapped to code sqrt(7): s = fl32(sqrt7 / g) with sqrt7 the fp32
 * value of sqrt(7); codes = clip(rint(fl32(z * s)), -8, 7), round half to even; d = fl32(g /
 * sqrt7).  Unlike absmax, values beyond 7/s are clipped.  pre (optional) = z * s in double, the
 * value the rounding decides on.
 */
void oracle_quant_act_absmean4(const float *z, int64_t M, int64_t K, int8_t *codes, float *d,
                               double *pre, int64_t *rowsum) {
    const float sqrt7 = (float)sqrt(7.0);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const float *row = z + m * K;
        double sa = 0.0;
        for (int64_t k = 0; k < K; ++k) sa += fabs((double)row[k]);
        double beta = sa / (double)K;
        float g = (float)(beta < 1e-5 ? 1e-5 : beta);
        volatile float s = sqrt7 / g;
        volatile float dq = g / sqrt7;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            volatile float v = row[k] * s;
            float t = nearbyintf(v);
            if (t > 7.0f) t = 7.0f;
            if (t < -8.0f) t = -8.0f;
            codes[m * K + k] = (int8_t)t;
            sum += (int64_t)t;
            if (pre) pre[m * K + k] = (double)row[k] * (double)s;
        }
        d[m] = dq;
        if (rowsum) rowsum[m] = sum;
    }
}

/* INT4 storage in HBM: every 8 consecutive codes k0..k0+7 fill one 32-bit word (4 bytes);
 * byte j (j in 0..3) holds code k0+j in its low nibble and code k0+4+j in its high nibble,
 * two's complement.  K must be a multiple of 8. */
void oracle_pack_int4(const int8_t *c, int64_t M, int64_t K, uint8_t *out) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k0 = 0; k0 < K; k0 += 8) {
            for (int j = 0; j < 4; ++j) {
                uint8_t lo = (uint8_t)(c[m * K + k0 + j] & 0x0F);
                uint8_t hi = (uint8_t)(c[m * K + k0 + 4 + j] & 0x0F);
                out[m * (K / 2) + k0 / 2 + j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

void oracle_unpack_int4(const uint8_t *in, int64_t M, int64_t K, int8_t *c) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k0 = 0; k0 < K; k0 += 8) {
            for (int j = 0; j < 4; ++j) {
                uint8_t b = in[m * (K / 2) + k0 / 2 + j];
                int lo = b & 0x0F, hi = b >> 4;
                c[m * K + k0 + j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
                c[m * K + k0 + 4 + j] = (int8_t)(hi >= 8 ? hi - 16 : hi);
            }
        }
    }
}

/* ------------------------------------------------------------------------------------- */
/* Step 4: ternary x integer product  [2B4T 一.2], [b1.58 技术贡献]                         */
/* ------------------------------------------------------------------------------------- */

/* acc[m][n] = sum_k c[m][k] * q[n][k] in int64 (c: [M][K] codes, q: [N][K] ternary). */
void oracle_gemm_i64(const int8_t *c, const int8_t *q, int64_t M, int64_t N, int64_t K,
                     int64_t *acc) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)c[m * K + k] * (int64_t)q[n * K + k];
            acc[m * N + n] = s;
        }
    }
}

/* The same product written the way the 2B4T article describes it: a weight of +1 adds the
 * activation, -1 subtracts it, 0 skips it.  No multiplications. */
void oracle_gemm_addsub(const int8_t *c, const int8_t *q, int64_t M, int64_t N, int64_t K,
                        int64_t *acc) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                int8_t w = q[n * K + k];
                if (w == 1) s += c[m * K + k];
                else if (w == -1) s -= c[m * K + k];
            }
            acc[m * N + n] = s;
        }
    }
}

/* ------------------------------------------------------------------------------------- */
/* Step 5: rescale to bf16                                                                 */
/* ------------------------------------------------------------------------------------- */

/* Y[m][n] = bf16_rn(acc[m][n] * d[m] * gamma), the product in double. */
void oracle_dequant(const int64_t *acc, const float *d, float gamma, int64_t M, int64_t N,
                    uint16_t *Y) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            Y[m * N + n] = double_to_bf16_rn((double)acc[m * N + n] * (double)d[m] * (double)gamma);
}

/* Activations fused after the rescale, for the up / gate projections that feed the FFN
 * [2B4T 一.3: squared ReLU activation], [v2: SwishGLU activation].  v = acc * d * gamma in
 * double, then
 *   act 1 (squared ReLU): Y[m][n] = bf16(max(v, 0)^2), N columns;
 *   act 2 (SwiGLU on interleaved rows, feature 2j the gate and 2j+1 the up projection):
 *         Y[m][j] = bf16(silu(v[2j]) * v[2j+1]), silu(x) = x / (1 + exp(-x)), N/2 columns.
 * The pages name the activations only; the interleaving is this library's layout. */
void oracle_dequant_act(const int64_t *acc, const float *d, float gamma, int64_t M, int64_t N,
                        int act, uint16_t *Y) {
    for (int64_t m = 0; m < M; ++m) {
        const double s = (double)d[m] * (double)gamma;
        if (act == 1) {
            for (int64_t n = 0; n < N; ++n) {
                const double v = (double)acc[m * N + n] * s;
                const double r = v > 0.0 ? v : 0.0;
                Y[m * N + n] = double_to_bf16_rn(r * r);
            }
        } else {
            for (int64_t j = 0; j < N / 2; ++j) {
                const double g = (double)acc[m * N + 2 * j] * s;
                const double u = (double)acc[m * N + 2 * j + 1] * s;
                Y[m * (N / 2) + j] = double_to_bf16_rn(g / (1.0 + exp(-g)) * u);
            }
        }
    }
}

/* ------------------------------------------------------------------------------------- */
/* Low-bit Q / K / V states  [v2, Tables 2 and 3]                                           */
/* ------------------------------------------------------------------------------------- */

/* The write-up's Tables 2 and 3 vary the bit width of the attention's Q, K and V states (a 3-bit
 * KV cache matches full precision); the quantiser's formula is not printed.  Reading: the
 * activations' absmax rule per token, or per group of `group` consecutive features of a token
 * (one attention head, group = head_dim), with Q = 2^(bits-1) - 1 (3 for 3 bits):
 *   m = max |x| over the group, s = Q / max(m, 1e-5) (fp32 IEEE), c = clip(rint(fl32(x * s)),
 *   -Q-1, Q) with round-half-even, d = max(m, 1e-5) / Q (fp32).
 * x holds the bf16 states widened to fp32 (exact).  codes: int8 [M][C]; d: [M][C / group];
 * pre (optional): x * Q / max(m, 1e-5) in double, the unrounded value.  C % group == 0. */
void oracle_quant_states(const float *x, int64_t M, int64_t C, int64_t group, int bits,
                         int8_t *codes, float *d, double *pre) {
    const float Q = (float)((1 << (bits - 1)) - 1);
    const float lo = -Q - 1.0f;
    const int64_t G = C / group;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            const float *row = x + m * C + g * group;
            float mx = 0.0f;
            for (int64_t k = 0; k < group; ++k) {
                float a = fabsf(row[k]);
                if (a > mx) mx = a;
            }
            float gm = mx < 1e-5f ? 1e-5f : mx;
            volatile float s = Q / gm;
            volatile float dq = gm / Q;
            for (int64_t k = 0; k < group; ++k) {
                volatile float v = row[k] * s;
                float t = nearbyintf(v);
                if (t > Q) t = Q;
                if (t < lo) t = lo;
                codes[m * C + g * group + k] = (int8_t)t;
                if (pre) pre[m * C + g * group + k] = (double)row[k] * (double)Q / (double)gm;
            }
            d[m * G + g] = dq;
        }
    }
}

/* Storage of `bits`-bit codes: each row is a little-endian bit stream, code k of the row in bits
 * bits*k .. bits*k + bits - 1 (two's complement), so a row takes C * bits / 8 bytes (C % 8 == 0).
 * unpack sign-extends back to int8. */
void oracle_pack_bits(const int8_t *c, int64_t M, int64_t C, int bits, uint8_t *out) {
    const int64_t rb = C * bits / 8;
    memset(out, 0, (size_t)(M * rb));
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < C; ++k) {
            const unsigned v = (unsigned)c[m * C + k] & ((1u << bits) - 1u);
            for (int b = 0; b < bits; ++b) {
                const int64_t bit = k * bits + b;
                if (v >> b & 1u) out[m * rb + bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
}

void oracle_unpack_bits(const uint8_t *in, int64_t M, int64_t C, int bits, int8_t *c) {
    const int64_t rb = C * bits / 8;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < C; ++k) {
            int v = 0;
            for (int b = 0; b < bits; ++b) {
                const int64_t bit = k * bits + b;
                v |= (in[m * rb + bit / 8] >> (bit % 8) & 1) << b;
            }
            if (v >> (bits - 1) & 1) v -= 1 << bits;
            c[m * C + k] = (int8_t)v;
        }
}

/* ------------------------------------------------------------------------------------- */
/* The whole forward, step by step                                                         */
/* ------------------------------------------------------------------------------------- */

/* Y = BitLinear(X) (hadamard == 0) or H-BitLinear(X) (hadamard != 0), from bf16 X [M][K] and
 * latent bf16 W [N][K].  bits = 8 quantises the tokens with absmax to INT8, bits = 4 with
 * absmean to INT4 (int4_absmax != 0: the absmax variant with Q = 7 instead).  Optional outputs
 * expose each stage: gamma, ternary q [N][K], the transformed activations z [M][K] (double,
 * before quantisation), codes [M][K], d [M], acc [M][N].  Returns 0, or -1 when a buffer
 * cannot be allocated. */
int oracle_bitlinear_forward_norm(const uint16_t *X, int64_t M, int64_t K, const uint16_t *W,
                                  int64_t N, int hadamard, int bits, int int4_absmax, int norm,
                                  const uint16_t *norm_gain, double norm_eps, uint16_t *Y,
                                  float *gamma_out, int8_t *q_out, double *z_out,
                                  int8_t *codes_out, float *d_out, int64_t *acc_out);

int oracle_bitlinear_forward(const uint16_t *X, int64_t M, int64_t K, const uint16_t *W,
                             int64_t N, int hadamard, int bits, uint16_t *Y,
                             float *gamma_out, int8_t *q_out, double *z_out,
                             int8_t *codes_out, float *d_out, int64_t *acc_out) {
    return oracle_bitlinear_forward_norm(X, M, K, W, N, hadamard, bits, 0, 0, NULL, 0.0, Y,
                                         gamma_out, q_out, z_out, codes_out, d_out, acc_out);
}

/* As oracle_bitlinear_forward; with norm != 0 each token row is RMS-normalised first
 * (oracle_rmsnorm with norm_gain and norm_eps) and the double result feeds the transform. */
int oracle_bitlinear_forward_norm(const uint16_t *X, int64_t M, int64_t K, const uint16_t *W,
                                  int64_t N, int hadamard, int bits, int int4_absmax, int norm,
                                  const uint16_t *norm_gain, double norm_eps, uint16_t *Y,
                                  float *gamma_out, int8_t *q_out, double *z_out,
                                  int8_t *codes_out, float *d_out, int64_t *acc_out) {
    int rc = -1;
    int8_t *q = malloc((size_t)(N * K));
    double *x = malloc((size_t)(M * K) * sizeof(double));
    double *z = malloc((size_t)(M * K) * sizeof(double));
    float *zf = malloc((size_t)(M * K) * sizeof(float));
    int8_t *c = malloc((size_t)(M * K));
    float *d = malloc((size_t)M * sizeof(float));
    int64_t *acc = malloc((size_t)(M * N) * sizeof(int64_t));
    if (!q || !x || !z || !zf || !c || !d || !acc) goto out;

    float gamma = oracle_absmean_gamma(W, N * K);
    oracle_ternarize(W, N * K, gamma, q);

    for (int64_t i = 0; i < M * K; ++i) x[i] = bf16_to_double(X[i]);
    if (norm) {
        oracle_rmsnorm(x, M, K, norm_gain, norm_eps, z);
        memcpy(x, z, (size_t)(M * K) * sizeof(double));
    }
    if (hadamard) oracle_fwht(x, M, K, z);
    else memcpy(z, x, (size_t)(M * K) * sizeof(double));
    for (int64_t i = 0; i < M * K; ++i) zf[i] = (float)z[i];

    if (bits == 4 && !int4_absmax) oracle_quant_act_absmean4(zf, M, K, c, d, NULL, NULL);
    else oracle_quant_act(zf, M, K, bits, c, d, NULL, NULL);
    oracle_gemm_i64(c, q, M, N, K, acc);
    oracle_dequant(acc, d, gamma, M, N, Y);

    if (gamma_out) *gamma_out = gamma;
    if (q_out) memcpy(q_out, q, (size_t)(N * K));
    if (z_out) memcpy(z_out, z, (size_t)(M * K) * sizeof(double));
    if (codes_out) memcpy(codes_out, c, (size_t)(M * K));
    if (d_out) memcpy(d_out, d, (size_t)M * sizeof(float));
    if (acc_out) memcpy(acc_out, acc, (size_t)(M * N) * sizeof(int64_t));
    rc = 0;
out:
    free(q); free(x); free(z); free(zf); free(c); free(d); free(acc);
    return rc;
}
