/*
 * mixllm_oracle.c -- plain, slow CPU oracle for the MixLLM W4.4A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header, table or constant
 * generator with the CUDA library: every value here is restated from the
 * sources below and written out in the plainest form.
 *
 * Sources (two of the web pages about the paper "MixLLM: LLM Quantization
 * with Global Mixed-precision between Output-features and Highly-efficient
 * System Design"):
 *   [NOTES] MLSys 2026 conference talk notes on MixLLM (notes.yuuk.io), in
 *           Japanese; sections are quoted by their headings.
 *   [WIKI]  awesome-system-papers summary "MixLLM ... (MLSys 2026)", in
 *           Chinese; sections are quoted by their headings.
 *
 * Arithmetic rules (compile with -ffp-contract=off, no fast-math):
 *   - fp32 IEEE operations in the order written below, no FMA contraction;
 *   - rounding to integer is round-half-to-even (nearbyintf in the default
 *     rounding mode); the pages only say "RTN" -- half-to-even is the
 *     reading taken, and the GPU side must make the same decision;
 *   - fp16 values are carried as their IEEE binary16 bit patterns (uint16_t)
 *     and converted with f32_to_f16_rne / f16_to_f32 below.
 *
 * Readings of points the pages leave open (each one is also a test pin):
 *   R1 activation scale s_a = amax/127, the IEEE fp32 quotient, kept as fp32;
 *      q = clamp(rne(x/s_a), -127, 127) with x/s_a the IEEE fp32 quotient; an
 *      all-zero group gets s_a = 0 and q = 0.  The pages give no dtype for this
 *      scale; fp32 is the plainest reading of "8-bit symmetric RTN".
 *   R2 4-bit asymmetric: lo = min(0, min w), hi = max(0, max w);
 *      s = fp16(min((hi-lo)/15, 65504)); if s == 0 the group is all zero
 *      (q = z = 0); else z = clamp(rne(-lo/s), 0, 15),
 *      q = clamp(rne(w/s) + z, 0, 15).
 *   R3 8-bit symmetric: s = fp16(min(amax/127, 65504)); if s == 0 then q = 0;
 *      else q = clamp(rne(w/s), -127, 127).
 *   R4 two-step GEMM: P = sum_{k in g} (Wq - z)*Aq in exact integers; then
 *      acc = acc + (float)P * (s_w * s_a), groups in ascending order, fp32;
 *      Y = fp16(acc).
 *   R5 channel salience: c_q is the channel's 4-bit asymmetric quantization
 *      (R2), dequantized as s*(q - z); the gradients are inputs; fp64.
 *   R6 top-T selection: equal saliences in list order (lower index first).
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_GROUP 128

/* ------------------------------------------------------------------ */
/* IEEE binary16 <-> binary32, written from the format definition.     */
/* ------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary16 -> binary32 (exact). */
float oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) & 1u;
    uint32_t exp = (uint32_t)(h >> 10) & 0x1Fu;
    uint32_t man = (uint32_t)h & 0x3FFu;
    float mag;
    if (exp == 0) {
        /* zero or subnormal: man * 2^-24 */
        mag = ldexpf((float)man, -24);
    } else if (exp == 31) {
        mag = man ? NAN : INFINITY;
    } else {
        /* (1024 + man) * 2^(exp - 25) */
        mag = ldexpf((float)(1024u + man), (int)exp - 25);
    }
    return sign ? -mag : mag;
}

/* binary32 -> binary16, round to nearest, ties to even; overflow -> inf. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    float a = fabsf(f);
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0f) return sign;
    /* Write a = m * 2^e with m in [1, 2). */
    int e;
    float m = frexpf(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    e -= 1;                   /* now a = (2m) * 2^e, 2m in [1, 2) */
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    /* Quantum of the target grid: 2^(e-10) for normals, 2^-24 below. */
    int qexp = (e >= -14) ? (e - 10) : -24;
    /* units of the quantum, exact in fp32 (a has 24 significant bits and the
     * quotient by a power of two is exact unless it underflows, which it
     * cannot here). */
    float units = ldexpf(a, -qexp);
    float r = nearbyintf(units); /* ties to even */
    uint32_t n = (uint32_t)r;
    (void)m;
    if (e >= -14) {
        /* normal range: n in [1024, 2048]; 2048 means carry into exponent */
        int ee = e;
        if (n == 2048u) { n = 1024u; ee += 1; }
        if (ee > 15) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | (uint16_t)((uint32_t)(ee + 15) << 10) | (uint16_t)(n - 1024u));
    }
    /* subnormal range: n in [0, 1024]; 1024 is the smallest normal, whose
     * bit pattern is exactly 0x0400, so the same formula holds. */
    return (uint16_t)(sign | (uint16_t)n);
}

/* Array form of the conversion (for the tests). */
void oracle_f32_to_f16_array(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(x[i]);
}

void oracle_f16_to_f32_array(const uint16_t *x, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(x[i]);
}

/* ------------------------------------------------------------------ */
/* Fast I2F ([NOTES] §高速 I2F 変換; [WIKI] 系统优化 "Fast I2F").        */
/* The bias 0x4b400000 is the float 1.5 * 2^23 = 12582912.0.  Adding it */
/* to an int32 P and reading the bits as float gives 12582912 + P for  */
/* every P with -2^22 <= P < 2^22.                                      */
/* ------------------------------------------------------------------ */

float oracle_i2f_bias(int32_t p)
{
    uint32_t biased = (uint32_t)p + 0x4b400000u;
    return bits_f32(biased) - 12582912.0f;
}

/* Number of P in [lo, hi) where the bias trick differs from (float)P. */
int64_t oracle_i2f_mismatches(int64_t lo, int64_t hi)
{
    int64_t bad = 0;
    for (int64_t p = lo; p < hi; ++p) {
        float a = oracle_i2f_bias((int32_t)p);
        float b = (float)(int32_t)p;
        if (f32_bits(a) != f32_bits(b)) ++bad;
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* Activation quantization: 8-bit symmetric, per token, group-wise RTN, */
/* group 128 ([NOTES] §設計判断の概要; [WIKI] 核心方法 "量化配置决策").     */
/* X, fp16 bits [M, K] row-major -> A_q int8 [M, K], s_a fp32 [M, K/128] */
/* ------------------------------------------------------------------ */

void oracle_quantize_act(const uint16_t *X, int64_t M, int64_t K,
                         int8_t *A_q, float *s_a)
{
    int64_t G = K / ORACLE_GROUP;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *x = X + m * K + g * ORACLE_GROUP;
            float amax = 0.0f;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                float v = fabsf(oracle_f16_to_f32(x[i]));
                if (v > amax) amax = v;
            }
            float s = amax / 127.0f;
            s_a[m * G + g] = s;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                int q = 0;
                if (s != 0.0f) {
                    float r = nearbyintf(oracle_f16_to_f32(x[i]) / s);
                    if (r > 127.0f) r = 127.0f;
                    if (r < -127.0f) r = -127.0f;
                    q = (int)r;
                }
                A_q[m * K + g * ORACLE_GROUP + i] = (int8_t)q;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* 4-bit asymmetric weight quantization, group 128 ([NOTES] §設計判断の概要,*/
/* "4-bit asymmetric, group size 128"; the zero point is a uint4, and a  */
/* uint4 minus a uint4 stays inside int8 -- [NOTES] §二段階逆量子化...).   */
/* W fp32 [N, K] -> q uint8 [N, K] (values 0..15, one per byte),        */
/*                  z uint8 [N, G] (0..15), s fp16 bits [N, G].          */
/* ------------------------------------------------------------------ */

void oracle_quantize_w4(const float *W, int64_t N, int64_t K,
                        uint8_t *q, uint8_t *z, uint16_t *s)
{
    int64_t G = K / ORACLE_GROUP;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + g * ORACLE_GROUP;
            float lo = 0.0f, hi = 0.0f;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                if (w[i] < lo) lo = w[i];
                if (w[i] > hi) hi = w[i];
            }
            float sc = (hi - lo) / 15.0f;
            if (sc > 65504.0f) sc = 65504.0f;
            uint16_t sh = oracle_f32_to_f16(sc);
            float sf = oracle_f16_to_f32(sh);
            int zi = 0;
            if (sf != 0.0f) {
                float zr = nearbyintf(-lo / sf);
                if (zr < 0.0f) zr = 0.0f;
                if (zr > 15.0f) zr = 15.0f;
                zi = (int)zr;
            }
            s[n * G + g] = sh;
            z[n * G + g] = (uint8_t)zi;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                int qi = 0;
                if (sf != 0.0f) {
                    float r = nearbyintf(w[i] / sf) + (float)zi;
                    if (r < 0.0f) r = 0.0f;
                    if (r > 15.0f) r = 15.0f;
                    qi = (int)r;
                }
                q[n * K + g * ORACLE_GROUP + i] = (uint8_t)qi;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* 8-bit symmetric weight quantization, group 128 ([WIKI] 核心方法:       */
/* "the 8-bit part is symmetric to simplify the kernel").                */
/* W fp32 [N, K] -> q int8 [N, K], s fp16 bits [N, G].                   */
/* ------------------------------------------------------------------ */

void oracle_quantize_w8(const float *W, int64_t N, int64_t K,
                        int8_t *q, uint16_t *s)
{
    int64_t G = K / ORACLE_GROUP;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + g * ORACLE_GROUP;
            float amax = 0.0f;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                float v = fabsf(w[i]);
                if (v > amax) amax = v;
            }
            float sc = amax / 127.0f;
            if (sc > 65504.0f) sc = 65504.0f;
            uint16_t sh = oracle_f32_to_f16(sc);
            float sf = oracle_f16_to_f32(sh);
            s[n * G + g] = sh;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                int qi = 0;
                if (sf != 0.0f) {
                    float r = nearbyintf(w[i] / sf);
                    if (r > 127.0f) r = 127.0f;
                    if (r < -127.0f) r = -127.0f;
                    qi = (int)r;
                }
                q[n * K + g * ORACLE_GROUP + i] = (int8_t)qi;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Channel split: the 8-bit set is the channels flagged in the global   */
/* bit map ([WIKI] 系统性缺陷, 可观测性与运维: a deployment asset); both sets */
/* are listed in ascending channel order (the order inside a set is not */
/* fixed by the pages; ascending is the reading taken).                 */
/* Returns N8.                                                           */
/* ------------------------------------------------------------------ */

int64_t oracle_split_channels(const uint8_t *is8, int64_t N,
                              int32_t *idx4, int32_t *idx8)
{
    int64_t n4 = 0, n8 = 0;
    for (int64_t n = 0; n < N; ++n) {
        if (is8[n]) idx8[n8++] = (int32_t)n;
        else idx4[n4++] = (int32_t)n;
    }
    return n8;
}

/* ------------------------------------------------------------------ */
/* Two-step dequantization GEMM ([NOTES] §二段階逆量子化による int8      */
/* Tensor Core 活用, steps 1-3; [NOTES] §並列実行 for the scatter of the  */
/* two channel sets into one output).                                    */
/*                                                                       */
/* Inputs in logical (unpacked) form:                                    */
/*   A_q int8 [M, K], s_a fp32 [M, G]                                    */
/*   4-bit set: q4 uint8 [N4, K] (0..15), z4 uint8 [N4, G],              */
/*              s4 fp16 bits [N4, G], idx4 int32 [N4]                    */
/*   8-bit set: q8 int8 [N8, K], s8 fp16 bits [N8, G], idx8 int32 [N8]   */
/* Output Y fp16 bits [M, N4 + N8]; column idx[n] receives channel n.    */
/* ------------------------------------------------------------------ */

static int32_t group_partial_w4(const int8_t *a, const uint8_t *q, int zp)
{
    int32_t p = 0;
    for (int i = 0; i < ORACLE_GROUP; ++i)
        p += ((int32_t)q[i] - (int32_t)zp) * (int32_t)a[i];
    return p;
}

static int32_t group_partial_w8(const int8_t *a, const int8_t *q)
{
    int32_t p = 0;
    for (int i = 0; i < ORACLE_GROUP; ++i)
        p += (int32_t)q[i] * (int32_t)a[i];
    return p;
}

void oracle_gemm_w4w8a8(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                        const uint8_t *q4, const uint8_t *z4, const uint16_t *s4,
                        const int32_t *idx4, int64_t N4,
                        const int8_t *q8, const uint16_t *s8,
                        const int32_t *idx8, int64_t N8,
                        uint16_t *Y)
{
    int64_t G = K / ORACLE_GROUP;
    int64_t N = N4 + N8;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N4; ++n) {
            float acc = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int32_t p = group_partial_w4(A_q + m * K + g * ORACLE_GROUP,
                                             q4 + n * K + g * ORACLE_GROUP,
                                             z4[n * G + g]);
                float scale = oracle_f16_to_f32(s4[n * G + g]) * s_a[m * G + g];
                acc = acc + (float)p * scale;
            }
            Y[m * N + idx4[n]] = oracle_f32_to_f16(acc);
        }
        for (int64_t n = 0; n < N8; ++n) {
            float acc = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int32_t p = group_partial_w8(A_q + m * K + g * ORACLE_GROUP,
                                             q8 + n * K + g * ORACLE_GROUP);
                float scale = oracle_f16_to_f32(s8[n * G + g]) * s_a[m * G + g];
                acc = acc + (float)p * scale;
            }
            Y[m * N + idx8[n]] = oracle_f32_to_f16(acc);
        }
    }
}

/* Per-group int32 partials P[m, idx[n], g] (step 2 alone, no bias). */
void oracle_group_partials(const int8_t *A_q, int64_t M, int64_t K,
                           const uint8_t *q4, const uint8_t *z4, const int32_t *idx4, int64_t N4,
                           const int8_t *q8, const int32_t *idx8, int64_t N8,
                           int32_t *P)
{
    int64_t G = K / ORACLE_GROUP;
    int64_t N = N4 + N8;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N4; ++n)
            for (int64_t g = 0; g < G; ++g)
                P[(m * N + idx4[n]) * G + g] =
                    group_partial_w4(A_q + m * K + g * ORACLE_GROUP,
                                     q4 + n * K + g * ORACLE_GROUP, z4[n * G + g]);
        for (int64_t n = 0; n < N8; ++n)
            for (int64_t g = 0; g < G; ++g)
                P[(m * N + idx8[n]) * G + g] =
                    group_partial_w8(A_q + m * K + g * ORACLE_GROUP,
                                     q8 + n * K + g * ORACLE_GROUP);
    }
}

/* ------------------------------------------------------------------ */
/* The library's packed weight layout, restated from its specification  */
/* (a storage format, so both sides must agree on it byte for byte):    */
/*   W4 bytes [ceil(N4/128)][G][128][64]: tile t, group g is one block  */
/*      of 128 rows (channels 128t .. 128t+127 of the 4-bit set; rows   */
/*      past N4 are zero) by the 64 bytes of the group's 128 codes; in  */
/*      each run of 32 consecutive k, byte i (0..15) holds element i in */
/*      its low nibble and element i+16 in its high nibble.             */
/*   z4 bytes [G, Np/2]: zero point of channel n, group g, in byte      */
/*      g*Np/2 + n/2, low nibble for even n, high nibble for odd n.     */
/*   s (either set) fp16 [G, Np]: scale of channel n, group g at g*Np+n. */
/*   Np = N rounded up to a multiple of 256; padding entries are zero.  */
/* ------------------------------------------------------------------ */

void oracle_pack_w4(const uint8_t *q, int64_t N4, int64_t K, uint8_t *W4)
{
    const int64_t G = K / 128, tiles = (N4 + 127) / 128;
    memset(W4, 0, (size_t)(tiles * G * 128 * 64));
    for (int64_t n = 0; n < N4; ++n) {
        const int64_t t = n / 128, r = n % 128;
        for (int64_t g = 0; g < G; ++g) {
            uint8_t *row = W4 + ((t * G + g) * 128 + r) * 64;
            for (int64_t run = 0; run < 4; ++run) {
                const int64_t base = g * 128 + run * 32;
                for (int i = 0; i < 16; ++i) {
                    uint8_t lo = q[n * K + base + i] & 0x0F;
                    uint8_t hi = q[n * K + base + 16 + i] & 0x0F;
                    row[run * 16 + i] = (uint8_t)(lo | (hi << 4));
                }
            }
        }
    }
}

void oracle_pack_zeros(const uint8_t *z, int64_t N, int64_t G, int64_t Np, uint8_t *z_packed)
{
    memset(z_packed, 0, (size_t)(G * Np / 2));
    for (int64_t g = 0; g < G; ++g)
        for (int64_t n = 0; n < N; ++n) {
            uint8_t v = z[n * G + g] & 0x0F;
            uint8_t *b = z_packed + g * (Np / 2) + n / 2;
            if (n % 2 == 0) *b = (uint8_t)((*b & 0xF0) | v);
            else *b = (uint8_t)((*b & 0x0F) | (v << 4));
        }
}

void oracle_pack_scales(const uint16_t *s, int64_t N, int64_t G, int64_t Np, uint16_t *s_packed)
{
    memset(s_packed, 0, (size_t)(G * Np) * sizeof(uint16_t));
    for (int64_t g = 0; g < G; ++g)
        for (int64_t n = 0; n < N; ++n)
            s_packed[g * Np + n] = s[n * G + g];
}

/* ------------------------------------------------------------------ */
/* Global mixed-precision search, step 1: the salience of every output  */
/* channel (MLSys 2026 talk notes on MixLLM, notes.yuuk.io,             */
/* §グローバル混合精度探索).  The loss change of quantizing channel c   */
/* alone, expanded to second order with the Fisher approximation of the */
/* Hessian, reduces to                                                  */
/*   S_c = (1/|D|) sum_d | g_d^T (c_q - c_0) + 1/2 (g_d^T (c_q - c_0))^2 | */
/* with g_d the gradient of the loss on sample d with respect to the    */
/* channel's weights, c_0 the channel's weights and c_q the channel     */
/* after quantization.  Reading taken: c_q is the low-bit form of the   */
/* layer, the 4-bit asymmetric group quantization of                    */
/* oracle_quantize_w4, dequantized as s * (q - z).                      */
/* W fp32 [N, K]; G fp32 [D, N, K]; S fp64 [N].  Everything in fp64.    */
/* ------------------------------------------------------------------ */
void oracle_channel_salience(const float *W, int64_t N, int64_t K, const float *G, int64_t D, double *S)
{
    const int64_t Gr = K / ORACLE_GROUP;
    uint8_t *q = (uint8_t *)malloc((size_t)(N * K));
    uint8_t *z = (uint8_t *)malloc((size_t)(N * Gr));
    uint16_t *s = (uint16_t *)malloc((size_t)(N * Gr) * sizeof(uint16_t));
    double *delta = (double *)malloc((size_t)K * sizeof(double));
    oracle_quantize_w4(W, N, K, q, z, s);
    for (int64_t n = 0; n < N; ++n) {
        /* c_q - c_0, exact in fp64 */
        for (int64_t k = 0; k < K; ++k) {
            const int64_t g = k / ORACLE_GROUP;
            const double cq = (double)oracle_f16_to_f32(s[n * Gr + g]) * (double)((int)q[n * K + k] - (int)z[n * Gr + g]);
            delta[k] = cq - (double)W[n * K + k];
        }
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) {
            const float *gd = G + (d * N + n) * K;
            double t = 0.0;
            for (int64_t k = 0; k < K; ++k) t += (double)gd[k] * delta[k];
            acc += fabs(t + 0.5 * t * t);
        }
        S[n] = D > 0 ? acc / (double)D : 0.0;
    }
    free(q);
    free(z);
    free(s);
    free(delta);
}

/* ------------------------------------------------------------------ */
/* Global mixed-precision search, step 2 (Algorithm 1 of the same      */
/* notes): all output channels of all layers in one list, sorted by    */
/* salience in descending order; the first T are given 8 bits.         */
/* Reading taken: equal saliences keep their list order (the lower     */
/* index first), so the set is unique.  S fp32 [Ntot] (both sides take */
/* this integer decision from the same fp32 keys); is8 [Ntot].         */
/* ------------------------------------------------------------------ */
static const float *g_sel_keys;
static int sel_cmp(const void *a, const void *b)
{
    const int64_t i = *(const int64_t *)a, j = *(const int64_t *)b;
    const float si = g_sel_keys[i], sj = g_sel_keys[j];
    if (si > sj) return -1;
    if (si < sj) return 1;
    return i < j ? -1 : (i > j ? 1 : 0);
}

void oracle_select_top_t(const float *S, int64_t Ntot, int64_t T, uint8_t *is8)
{
    int64_t *order = (int64_t *)malloc((size_t)(Ntot > 0 ? Ntot : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < Ntot; ++i) order[i] = i;
    g_sel_keys = S;
    qsort(order, (size_t)Ntot, sizeof(int64_t), sel_cmp);
    for (int64_t i = 0; i < Ntot; ++i) is8[i] = 0;
    for (int64_t r = 0; r < T && r < Ntot; ++r) is8[order[r]] = 1;
    free(order);
}
