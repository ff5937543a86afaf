/*
 * w4_oracle.c -- plain CPU oracle for group-wise INT4 weight quantization and
 * W4A16 inference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * under int4_w4a16_b200/) includes, links or calls this file.  Only tests/,
 * the smoke check in __graft_entry__.py and the cpu_baseline / reference arm
 * of bench.py load it.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Every function is the plain definition of what the method computes, in the
 * order the sources state it, with no blocking, fusion or reordering.  Loops
 * over independent rows may run on several OpenMP threads; the arithmetic of
 * each output element is the same sequential code whatever the thread count.
 *
 * Sources (cited by page title and section):
 *   [QAT]  SGLang RL team, "INT4 QAT end-to-end" blog (re-post): fake
 *          quantization + STE in Megatron (_FakeInt4QuantizationSTE), the
 *          [-7, 7] simulated INT4 range, Fig. 4 "Rollout-side INT4 weight
 *          only" (8 INT4 values packed into one INT32, 8 x 4 bits = 32 bits,
 *          pack_int4_to_int32), moe_align_block_size, "MoE operator deep
 *          fusion".
 *   [TAG]  reportify.cn concept page "量化感知训练" (quantization-aware
 *          training): para. [8][9] fake quant forward / STE backward,
 *          [10] real quantization of the exported weights, [11] 1x32 scale
 *          granularity, [32] two 4-bit weights per byte, [35]
 *          moe_align_block_size.
 *   [BAS]  "量化基础：从 FP32 到 INT4 的压缩艺术" (quantization basics):
 *          §1.3 table (INT4 range [-8, 7], BF16 = 1+8+7 bits),
 *          §2.2 symmetric quantization s = max|x| / q_max,
 *               q = clamp(round(x / s), -q_max, q_max),
 *          §2.4 error bound |x_hat - x| <= s/2,
 *          §6.1 numpy symmetric quantizer and its printed output,
 *          §6.2 torch.round rounds half to even.
 *
 * Readings where the sources are silent:
 *   - groups are 32 contiguous elements along K (the reduction dim) of a
 *     row-major [rows, K] BF16 matrix ([TAG] [11] "1x32");
 *   - s32 = fl32(amax / 7) in IEEE fp32, then s = bf16_rne(s32) is the
 *     stored scale, and q divides by that stored BF16 scale, so that fake
 *     quantization and dequantized export agree bit for bit;
 *   - q = clamp(rint_half_even(fl32(w / s)), -8, 7); with this scale the clamp
 *     never fires, so the [-7, 7] and [-8, 7] readings coincide;
 *   - amax == 0 or s rounding to 0 gives s = +0 and q = 0 for the group;
 *   - Wdq = bf16_rne(q * s), +0.0 when q == 0;
 *   - packing is low nibble first, two's complement nibbles, along K;
 *   - moe_align: stable sort of (token, k) slots by expert, runs padded to a
 *     multiple of the block size, sentinel T*topk, expert id -1 past the end.
 *
 * Inputs are assumed finite (NaN / Inf behaviour is unspecified).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* BF16 <-> FP32 ([BAS] §1.3: BF16 is 1 sign, 8 exponent, 7 mantissa bits,  */
/* i.e. the upper half of an IEEE fp32).                                     */
/* ------------------------------------------------------------------------ */

float w4o_f32_from_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round an fp32 to the nearest BF16, ties to even (finite inputs). */
uint16_t w4o_bf16_from_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

void w4o_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int w4o_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Group-32 symmetric INT4 quantization ([QAT] fake quantization / real      */
/* quantization; [BAS] §2.2 with q_max = 7 and the INT4 clamp of §1.3).      */
/* ------------------------------------------------------------------------ */

/* One group: returns the stored BF16 scale and writes q[0..n-1]. */
static uint16_t quantize_one_group(const uint16_t *w, int64_t n, int8_t *q)
{
    /* step 1: amax = max |w| over the group, on the BF16 values */
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(w4o_f32_from_bf16(w[i]));
        if (a > amax) amax = a;
    }
    /* step 2: s32 = amax / 7 in IEEE fp32 */
    volatile float seven = 7.0f;
    float s32 = amax / seven;
    /* step 3: the stored scale is BF16 */
    uint16_t s_bits = w4o_bf16_from_f32(s32);
    float s = w4o_f32_from_bf16(s_bits);
    /* step 4: q = clamp(round_half_even(w / s), -8, 7); q = 0 when s == 0 */
    for (int64_t i = 0; i < n; ++i) {
        if (s == 0.0f) {
            q[i] = 0;
            continue;
        }
        float y = w4o_f32_from_bf16(w[i]) / s;      /* IEEE fp32 quotient */
        float r = nearbyintf(y);                     /* default mode: ties to even */
        if (r < -8.0f) r = -8.0f;
        if (r > 7.0f) r = 7.0f;
        q[i] = (int8_t)r;
    }
    return s_bits;
}

/* q[rows*K] int8 codes and S[rows*(K/group)] BF16 scales. */
void w4o_quantize(const uint16_t *W, int64_t rows, int64_t K, int64_t group,
                  int8_t *q, uint16_t *S)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < gpr; ++g) {
            int64_t base = r * K + g * group;
            S[r * gpr + g] = quantize_one_group(W + base, group, q + base);
        }
}

/* Dequantized value of one code: bf16_rne(q * s), +0.0 for q == 0. */
static uint16_t dequant_one(int8_t q, uint16_t s_bits)
{
    float s = w4o_f32_from_bf16(s_bits);
    float v = (float)q * s;          /* exact in fp32: <= 4 x 8 significant bits */
    if (v == 0.0f) v = 0.0f;         /* +0.0 */
    return w4o_bf16_from_f32(v);
}

/* Fake quantization (quantize then immediately dequantize, storage stays BF16):
 * Wdq[rows*K]; S may be NULL. */
void w4o_fake_quant(const uint16_t *W, int64_t rows, int64_t K, int64_t group,
                    uint16_t *Wdq, uint16_t *S)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int8_t *qg = (int8_t *)malloc((size_t)group);
        for (int64_t g = 0; g < gpr; ++g) {
            int64_t base = r * K + g * group;
            uint16_t s_bits = quantize_one_group(W + base, group, qg);
            if (S) S[r * gpr + g] = s_bits;
            for (int64_t i = 0; i < group; ++i)
                Wdq[base + i] = dequant_one(qg[i], s_bits);
        }
        free(qg);
    }
}

/* Straight-through estimator backward: the gradient passes through the
 * rounding unchanged ([QAT] §2.1; [TAG] [9][17]). */
void w4o_ste_backward(const uint16_t *dWdq, int64_t n, uint16_t *dW)
{
    for (int64_t i = 0; i < n; ++i) dW[i] = dWdq[i];
}

/* ------------------------------------------------------------------------ */
/* Packing ([QAT] Fig. 4: eight INT4 values in one INT32; element i of the   */
/* eight sits at bits [4i, 4i+3] as a two's-complement nibble).              */
/* ------------------------------------------------------------------------ */

int32_t w4o_pack8(const int8_t *q8)
{
    uint32_t word = 0;
    for (int i = 0; i < 8; ++i)
        word |= ((uint32_t)q8[i] & 0xFu) << (4 * i);
    return (int32_t)word;
}

void w4o_unpack8(int32_t word, int8_t *q8)
{
    uint32_t u = (uint32_t)word;
    for (int i = 0; i < 8; ++i) {
        int v = (int)((u >> (4 * i)) & 0xFu);
        q8[i] = (int8_t)(v >= 8 ? v - 16 : v);
    }
}

void w4o_pack(const int8_t *q, int64_t n, int32_t *words)
{
    for (int64_t j = 0; j < n / 8; ++j) words[j] = w4o_pack8(q + 8 * j);
}

void w4o_unpack(const int32_t *words, int64_t n, int8_t *q)
{
    for (int64_t j = 0; j < n / 8; ++j) w4o_unpack8(words[j], q + 8 * j);
}

/* Real quantization for export: codes packed along K into Wq[rows*(K/8)]
 * plus BF16 scales S[rows*(K/group)]. */
void w4o_quantize_pack(const uint16_t *W, int64_t rows, int64_t K, int64_t group,
                       int32_t *Wq, uint16_t *S)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int8_t *qrow = (int8_t *)malloc((size_t)K);
        for (int64_t g = 0; g < gpr; ++g)
            S[r * gpr + g] = quantize_one_group(W + r * K + g * group, group,
                                                qrow + g * group);
        w4o_pack(qrow, K, Wq + r * (K / 8));
        free(qrow);
    }
}

/* Inverse of the export: unpack the codes and dequantize them. */
void w4o_dequant(const int32_t *Wq, const uint16_t *S, int64_t rows, int64_t K,
                 int64_t group, uint16_t *Wdq)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int8_t *qrow = (int8_t *)malloc((size_t)K);
        w4o_unpack(Wq + r * (K / 8), K, qrow);
        for (int64_t k = 0; k < K; ++k)
            Wdq[r * K + k] = dequant_one(qrow[k], S[r * gpr + k / group]);
        free(qrow);
    }
}

/* ------------------------------------------------------------------------ */
/* Group-32 asymmetric (zero-point) INT4 quantization: the affine map of     */
/* [BAS] §2.1 (q = clamp(round(x / s) + z, q_min, q_max), x^ = (q - z) * s)  */
/* with the asymmetric scale and zero point of [BAS] §2.3                    */
/* (s = (x_max - x_min) / (q_max - q_min), z = clamp(round(q_min - x_min/s)))*/
/* over the unsigned INT4 range q_min = 0, q_max = 15.  x_max and x_min are  */
/* the group's own extremes; the scale is stored in BF16 like the symmetric  */
/* one, the zero point as one byte per group.  A group with s == 0 (all      */
/* values equal) gets q = z = 0.                                             */
/* ------------------------------------------------------------------------ */

static uint16_t quantize_one_group_zp(const uint16_t *w, int64_t n, uint8_t *q,
                                      uint8_t *z_out)
{
    /* step 1: the group's extremes, on the BF16 values */
    float xmax = w4o_f32_from_bf16(w[0]), xmin = xmax;
    for (int64_t i = 1; i < n; ++i) {
        float x = w4o_f32_from_bf16(w[i]);
        if (x > xmax) xmax = x;
        if (x < xmin) xmin = x;
    }
    /* step 2: s = (x_max - x_min) / 15 in IEEE fp32, stored as BF16 */
    volatile float fifteen = 15.0f;
    float range = xmax - xmin;
    float s32 = range / fifteen;
    uint16_t s_bits = w4o_bf16_from_f32(s32);
    const float s = w4o_f32_from_bf16(s_bits);
    if (s == 0.0f) {
        for (int64_t i = 0; i < n; ++i) q[i] = 0;
        *z_out = 0;
        return s_bits;
    }
    /* step 3: z = clamp(round_half_even(0 - x_min / s), 0, 15) */
    float zf = nearbyintf(0.0f - xmin / s);
    if (zf < 0.0f) zf = 0.0f;
    if (zf > 15.0f) zf = 15.0f;
    /* step 4: q = clamp(round_half_even(x / s) + z, 0, 15) */
    for (int64_t i = 0; i < n; ++i) {
        float y = w4o_f32_from_bf16(w[i]) / s;      /* IEEE fp32 quotient */
        float v = nearbyintf(y) + zf;
        if (v < 0.0f) v = 0.0f;
        if (v > 15.0f) v = 15.0f;
        q[i] = (uint8_t)v;
    }
    *z_out = (uint8_t)zf;
    return s_bits;
}

/* q[rows*K] codes in [0, 15], S[rows*(K/group)] BF16 scales, Z zero points. */
void w4o_quantize_zp(const uint16_t *W, int64_t rows, int64_t K, int64_t group,
                     uint8_t *q, uint16_t *S, uint8_t *Z)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < gpr; ++g) {
            int64_t base = r * K + g * group;
            S[r * gpr + g] = quantize_one_group_zp(W + base, group, q + base, Z + r * gpr + g);
        }
}

/* Dequantized value of one code: bf16_rne((q - z) * s), +0.0 for q == z.
 * (q - z) * s is exact in fp32 (4 x 8 significant bits); the BF16 rounding
 * is the one step that can round. */
static uint16_t dequant_one_zp(uint8_t q, uint8_t z, uint16_t s_bits)
{
    float s = w4o_f32_from_bf16(s_bits);
    float v = (float)((int)q - (int)z) * s;
    if (v == 0.0f) v = 0.0f;
    return w4o_bf16_from_f32(v);
}

/* Eight unsigned codes <-> one word, element i at bits [4i, 4i+3]. */
int32_t w4o_pack8_u(const uint8_t *q8)
{
    uint32_t word = 0;
    for (int i = 0; i < 8; ++i)
        word |= (uint32_t)(q8[i] & 0xFu) << (4 * i);
    return (int32_t)word;
}

void w4o_unpack8_u(int32_t word, uint8_t *q8)
{
    uint32_t u = (uint32_t)word;
    for (int i = 0; i < 8; ++i) q8[i] = (uint8_t)((u >> (4 * i)) & 0xFu);
}

/* Export: Wq[rows*(K/8)] packed unsigned codes, S BF16 scales, Z zero points. */
void w4o_quantize_pack_zp(const uint16_t *W, int64_t rows, int64_t K, int64_t group,
                          int32_t *Wq, uint16_t *S, uint8_t *Z)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        uint8_t *qrow = (uint8_t *)malloc((size_t)K);
        for (int64_t g = 0; g < gpr; ++g)
            S[r * gpr + g] = quantize_one_group_zp(W + r * K + g * group, group,
                                                   qrow + g * group, Z + r * gpr + g);
        for (int64_t j = 0; j < K / 8; ++j) Wq[r * (K / 8) + j] = w4o_pack8_u(qrow + 8 * j);
        free(qrow);
    }
}

void w4o_dequant_zp(const int32_t *Wq, const uint16_t *S, const uint8_t *Z, int64_t rows,
                    int64_t K, int64_t group, uint16_t *Wdq)
{
    int64_t gpr = K / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        uint8_t q8[8];
        for (int64_t j = 0; j < K / 8; ++j) {
            w4o_unpack8_u(Wq[r * (K / 8) + j], q8);
            for (int i = 0; i < 8; ++i) {
                int64_t k = 8 * j + i;
                int64_t g = r * gpr + k / group;
                Wdq[r * K + k] = dequant_one_zp(q8[i], Z[g], S[g]);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Micro-scaled 4-bit floating point (the MR-GPTQ / QuTLASS summary page:    */
/* MXFP4 shares one scale per 32 elements, 4.25 bits per element, so an      */
/* 8-bit power-of-two scale; NVFP4 shares one per 16 elements).  The element */
/* format is the 4-bit float E2M1 (1 sign, 2 exponent bits with bias 1, 1     */
/* mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no inf or NaN).      */
/* Readings where the page is silent:                                        */
/*   - element rounding: nearest E2M1 value, ties to the even code (mantissa  */
/*     bit 0), magnitudes above 6 saturate to 6, zero is +0;                  */
/*   - MXFP4: scale 2^e with e = floor(log2(amax)) - 2 (2 = the exponent of   */
/*     E2M1's largest value), clamped to [-127, 127], stored as e + 127; an   */
/*     all-zero group stores e = 0;                                          */
/*   - NVFP4: an FP8 E4M3 group scale (bias 7, largest 448) under one fp32    */
/*     per-tensor scale g = fl32(amax_tensor / (6 * 448)) (g = 1 for an all-  */
/*     zero tensor); the group scale is amax_group / (6 g) rounded to E4M3    */
/*     (nearest, ties to the even code, saturating at 448); elements divide   */
/*     by s * g; a group whose scale rounds to 0 stores zeros;               */
/*   - dequantized value: bf16_rne(fl32(fl32(value(q) * s) * g)) (MXFP4:       */
/*     value(q) * 2^e, exact, then BF16).                                    */
/* Quotients are taken in fp64: a BF16 value over a 4- or 8-bit significand */
/* (times the fp32 g) is either exactly on a rounding midpoint or at least    */
/* 2^-32 relative away from it, far above the fp64 rounding error.           */
/* ------------------------------------------------------------------------ */

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double w4o_e2m1_value(uint8_t code)
{
    double v = kE2M1[code & 7u];
    return (code & 8u) ? -v : v;
}

/* Nearest-even rounding of v onto a sorted table of n non-negative values
 * (index order = code order), saturating at the last entry. */
static int round_to_table(double a, const double *tab, int n)
{
    if (a >= tab[n - 1]) return n - 1;
    int i = 0;
    while (i + 1 < n && tab[i + 1] <= a) ++i;       /* tab[i] <= a < tab[i+1] */
    if (a == tab[i]) return i;
    double lo = a - tab[i], hi = tab[i + 1] - a;
    if (lo < hi) return i;
    if (hi < lo) return i + 1;
    return (i % 2 == 0) ? i : i + 1;                 /* tie: the even code */
}

uint8_t w4o_e2m1_encode(double v)
{
    int c = round_to_table(fabs(v), kE2M1, 8);
    return (uint8_t)((c != 0 && v < 0.0) ? (c | 8) : c);
}

/* E4M3: code = e << 3 | m (positive half; 0x7F is NaN and never produced). */
double w4o_e4m3_value(uint8_t code)
{
    int e = (code >> 3) & 15, m = code & 7;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (code & 0x80u) ? -v : v;
}

uint8_t w4o_e4m3_encode(double v)      /* v >= 0 */
{
    static double tab[127];
    static int init = 0;
    if (!init) {
        for (int c = 0; c < 127; ++c) tab[c] = w4o_e4m3_value((uint8_t)c);
        init = 1;
    }
    return (uint8_t)round_to_table(v, tab, 127);
}

void w4o_quantize_mxfp4(const uint16_t *W, int64_t rows, int64_t K, uint8_t *q, uint8_t *E)
{
    int64_t gpr = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < gpr; ++g) {
            const uint16_t *w = W + r * K + g * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)w4o_f32_from_bf16(w[i]));
                if (a > amax) amax = a;
            }
            int e = 0;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex);                  /* amax = f * 2^ex, f in [0.5, 1) */
                e = (ex - 1) - 2;                  /* floor(log2(amax)) - 2 */
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            E[r * gpr + g] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i)
                q[r * K + g * 32 + i] =
                    amax > 0.0 ? w4o_e2m1_encode(ldexp((double)w4o_f32_from_bf16(w[i]), -e)) : 0;
        }
}

void w4o_dequant_mxfp4(const uint8_t *q, const uint8_t *E, int64_t rows, int64_t K,
                       uint16_t *Wdq)
{
    int64_t gpr = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double v = ldexp(w4o_e2m1_value(q[r * K + k]), (int)E[r * gpr + k / 32] - 127);
            float f = (float)v;                      /* exact: 2 bits times a power of two */
            if (f == 0.0f) f = 0.0f;
            Wdq[r * K + k] = w4o_bf16_from_f32(f);
        }
}

void w4o_quantize_nvfp4(const uint16_t *W, int64_t rows, int64_t K, uint8_t *q, uint8_t *S,
                        float *g_out)
{
    double amax_t = 0.0;
    for (int64_t i = 0; i < rows * K; ++i) {
        double a = fabs((double)w4o_f32_from_bf16(W[i]));
        if (a > amax_t) amax_t = a;
    }
    volatile float denom = 2688.0f;                  /* 6 * 448 */
    float g = amax_t > 0.0 ? (float)amax_t / denom : 1.0f;
    if (g == 0.0f) g = 1.0f;
    *g_out = g;
    int64_t gpr = K / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < gpr; ++j) {
            const uint16_t *w = W + r * K + j * 16;
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) {
                double a = fabs((double)w4o_f32_from_bf16(w[i]));
                if (a > amax) amax = a;
            }
            uint8_t sc = w4o_e4m3_encode(amax / (6.0 * (double)g));
            S[r * gpr + j] = sc;
            double step = w4o_e4m3_value(sc) * (double)g;
            for (int i = 0; i < 16; ++i)
                q[r * K + j * 16 + i] =
                    step > 0.0 ? w4o_e2m1_encode((double)w4o_f32_from_bf16(w[i]) / step) : 0;
        }
}

void w4o_dequant_nvfp4(const uint8_t *q, const uint8_t *S, float g, int64_t rows, int64_t K,
                       uint16_t *Wdq)
{
    int64_t gpr = K / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            float qs = (float)(w4o_e2m1_value(q[r * K + k]) *
                               w4o_e4m3_value(S[r * gpr + k / 16]));   /* exact */
            float f = qs * g;
            if (f == 0.0f) f = 0.0f;
            Wdq[r * K + k] = w4o_bf16_from_f32(f);
        }
}

/* ------------------------------------------------------------------------ */
/* Generic symmetric quantizer of [BAS] §2.2 / §6.1, in fp64, with the scale */
/* left unrounded: s = max|x| / qmax per group, q = clip(round(x/s)).       */
/* Used to reproduce the page's worked INT8 example.                         */
/* ------------------------------------------------------------------------ */
void w4o_symmetric_quantize_f64(const double *x, int64_t n, int64_t group,
                                int qmax, int32_t *q, double *s_out)
{
    for (int64_t g0 = 0, gi = 0; g0 < n; g0 += group, ++gi) {
        int64_t len = (n - g0 < group) ? n - g0 : group;
        double amax = 0.0;
        for (int64_t i = 0; i < len; ++i)
            if (fabs(x[g0 + i]) > amax) amax = fabs(x[g0 + i]);
        double s = amax / (double)qmax;
        s_out[gi] = s;
        for (int64_t i = 0; i < len; ++i) {
            double r = (s == 0.0) ? 0.0 : nearbyint(x[g0 + i] / s);
            if (r < -qmax) r = -qmax;
            if (r > qmax) r = qmax;
            q[g0 + i] = (int32_t)r;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* W4A16 GEMM: Y = X . dq(W)^T, FP32 accumulation in ascending k, one BF16   */
/* rounding of the result.  R (optional) receives the fp32 sums.             */
/* ------------------------------------------------------------------------ */
void w4o_gemm(const uint16_t *X, const uint16_t *Wdq, int64_t M, int64_t N,
              int64_t K, uint16_t *Y, float *R)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float prod = w4o_f32_from_bf16(X[m * K + k]) *
                             w4o_f32_from_bf16(Wdq[n * K + k]);   /* exact */
                acc = acc + prod;
            }
            if (R) R[m * N + n] = acc;
            if (Y) Y[m * N + n] = w4o_bf16_from_f32(acc);
        }
}

/* Same product, read straight from the packed export (unpack + dequant of one
 * row of W at a time, then the plain dot products). */
void w4o_w4a16_gemm(const uint16_t *X, const int32_t *Wq, const uint16_t *S,
                    int64_t M, int64_t N, int64_t K, int64_t group,
                    uint16_t *Y, float *R)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint16_t *wrow = (uint16_t *)malloc((size_t)K * sizeof(uint16_t));
        w4o_dequant(Wq + n * (K / 8), S + n * (K / group), 1, K, group, wrow);
        for (int64_t m = 0; m < M; ++m) {
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k)
                acc = acc + w4o_f32_from_bf16(X[m * K + k]) *
                            w4o_f32_from_bf16(wrow[k]);
            if (R) R[m * N + n] = acc;
            if (Y) Y[m * N + n] = w4o_bf16_from_f32(acc);
        }
        free(wrow);
    }
}

/* ------------------------------------------------------------------------ */
/* moe_align_block_size ([QAT] "merge and align the tokens of the same       */
/* expert"; [TAG] [35]).  Slot i = t*topk + k routes to e_i = topk_ids[i].   */
/* Each expert's slots, in ascending slot order, form one run padded up to   */
/* a multiple of `block`; runs follow in ascending expert id.  Padding and   */
/* everything past the padded total hold the sentinel T*topk; expert_ids is  */
/* the expert of each block, -1 past the end.  Slots whose expert id is out  */
/* of [0, E) are skipped.  Returns 0, or -1 if `cap` is too small.           */
/* ------------------------------------------------------------------------ */
int w4o_moe_align(const int32_t *topk_ids, int64_t T, int64_t topk, int64_t E,
                  int64_t block, int32_t *sorted_ids, int64_t cap,
                  int32_t *expert_ids, int32_t *num_post_pad)
{
    int64_t slots = T * topk;
    int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t i = 0; i < slots; ++i) {
        int32_t e = topk_ids[i];
        if (e >= 0 && e < E) cnt[e] += 1;
    }
    int64_t total = 0;
    for (int64_t e = 0; e < E; ++e)
        total += (cnt[e] + block - 1) / block * block;
    if (total > cap) {
        free(cnt);
        return -1;
    }
    for (int64_t p = 0; p < cap; ++p) sorted_ids[p] = (int32_t)slots;
    for (int64_t b = 0; b < cap / block; ++b) expert_ids[b] = -1;
    int64_t off = 0;
    for (int64_t e = 0; e < E; ++e) {
        int64_t r = 0;
        for (int64_t i = 0; i < slots; ++i)       /* ascending slot order */
            if (topk_ids[i] == e) sorted_ids[off + r++] = (int32_t)i;
        int64_t padded = (cnt[e] + block - 1) / block * block;
        for (int64_t b = off / block; b < (off + padded) / block; ++b)
            expert_ids[b] = (int32_t)e;
        off += padded;
    }
    *num_post_pad = (int32_t)total;
    free(cnt);
    return 0;
}

/* Grouped W4A16 GEMM over the aligned slot list: for every block b with
 * expert e and every real slot in it, C[slot, :] = A[slot / a_row_div, :] .
 * dq(W_e)^T, with the same fp32 accumulation as w4o_gemm.  Wdq holds every
 * expert's dequantized weights, [E, N, K].  Padding slots are not written. */
void w4o_moe_gemm(const uint16_t *A, int64_t a_row_div, const uint16_t *Wdq,
                  const int32_t *sorted_ids, const int32_t *expert_ids,
                  int64_t num_post_pad, int64_t num_slots, int64_t block,
                  int64_t N, int64_t K, uint16_t *C, float *R)
{
    #pragma omp parallel for schedule(dynamic)
    for (int64_t p = 0; p < num_post_pad; ++p) {
        int32_t slot = sorted_ids[p];
        int32_t e = expert_ids[p / block];
        if (slot < 0 || slot >= num_slots || e < 0) continue;
        const uint16_t *a = A + (int64_t)(slot / a_row_div) * K;
        const uint16_t *w = Wdq + (int64_t)e * N * K;
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k)
                acc = acc + w4o_f32_from_bf16(a[k]) * w4o_f32_from_bf16(w[n * K + k]);
            if (R) R[(int64_t)slot * N + n] = acc;
            if (C) C[(int64_t)slot * N + n] = w4o_bf16_from_f32(acc);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router gating ([QAT] the fused gating kernel before moe_align; its exact */
/* rule is silent, read as): p = softmax(logits) per token in fp32, the     */
/* topk largest p in descending order with ties to the lower expert id,     */
/* weights = the selected p (not renormalized).  The order is taken on the  */
/* logits, which is the order of the exact p (exp is strictly increasing).  */
/* ------------------------------------------------------------------------ */
void w4o_moe_gate_topk(const float *logits, int64_t T, int64_t E, int64_t topk,
                       int32_t *topk_ids, float *topk_weights)
{
    #pragma omp parallel for
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        float mx = l[0];
        for (int64_t e = 1; e < E; ++e) mx = l[e] > mx ? l[e] : mx;
        float sum = 0.0f;
        for (int64_t e = 0; e < E; ++e) sum = sum + expf(l[e] - mx);
        unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
        for (int64_t k = 0; k < topk; ++k) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)        /* strict >: ties keep the lower id */
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            topk_ids[t * topk + k] = (int32_t)best;
            topk_weights[t * topk + k] = expf(l[best] - mx) / sum;
        }
        free(taken);
    }
}

/* Weighted top-k combine after the down projection:
 * out[t, n] = bf16( sum_k w[t, k] * D[t*topk + k, n] ), fp32, ascending k,
 * each product rounded to fp32 before its add. */
void w4o_moe_combine(const uint16_t *D, const float *w, int64_t T, int64_t topk,
                     int64_t N, uint16_t *out)
{
    #pragma omp parallel for
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t k = 0; k < topk; ++k) {
                float prod = w[t * topk + k] * w4o_f32_from_bf16(D[(t * topk + k) * N + n]);
                acc = acc + prod;
            }
            out[t * N + n] = w4o_bf16_from_f32(acc);
        }
}
