// w4_qdq.cuh -- per-group quantize / dequantize arithmetic of the library's
// quantizers (w4_quant.cu), shared with the GEMM whose weight prologue runs the
// same QDQ on the fly (w4_gemm.cu, QAT forward).  The method: for a group of 32
// BF16 weights, s = bf16_rne(fl32(amax / 7)), q = clamp(rint_even(w / s), -8, 7),
// dq = bf16_rne(q * s) (INT4 QAT blog, fake quantization; reportify.cn
// "量化感知训练" [8][16]; "量化基础" §2.2).  The division-free exact rounding
// is described in w4_quant.cu.
#pragma once

#include "w4_common.cuh"

namespace w4 {
namespace qdq {

constexpr float kSnap = 12288.0f;         // 1.5 * 2^13: ulp 2^-10 around it
constexpr float kToInt = 12570624.0f;     // 1.5 * 2^23 - 1.5 * 2^13 (exact in fp32)
constexpr float kMagic = 12582912.0f;     // 1.5 * 2^23: ulp 1 around it

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// max(|a|, |b|) per BF16 half (the sign bit of each half is the XOR of the
// inputs' signs and is masked off by the caller).
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// amax of a group of 32 BF16 values (16 words); returns the BF16 bits of amax.
// The max of BF16 magnitudes is exact, and non-negative BF16 values order like
// their bit patterns.
__device__ __forceinline__ uint32_t group_amax_bits(const uint32_t (&v)[16]) {
    uint32_t m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = absmax2(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int j = 0; j < 4; ++j) m[j] = absmax2(m[2 * j], m[2 * j + 1]);
    m[0] = absmax2(absmax2(m[0], m[1]), absmax2(m[2], m[3])) & 0x7FFF7FFFu;
    return max(m[0] & 0xFFFFu, m[0] >> 16);
}

struct GroupScale {
    float s;        // the stored BF16 scale, widened
    float r;        // rcp.approx(s) on the fast path (relative error <= 2^-23)
    uint16_t bits;  // BF16 bits of s
    int mode;       // 0: s == 0, 1: normal s (fast path), 2: subnormal s
};

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ GroupScale make_scale(uint32_t amax_bits) {
    GroupScale g;
    const float a = __uint_as_float(amax_bits << 16);
    // fl32(a / 7) by one refinement step (exact for every BF16 a)
    const float c = __uint_as_float(0x3E124925u);     // fl32(1/7)
    const float q0 = __fmul_rn(a, c);
    const float rr = __fmaf_rn(-q0, 7.0f, a);
    const float s32 = __fmaf_rn(rr, c, q0);
    const __nv_bfloat16 sb = __float2bfloat16_rn(s32);
    g.bits = *reinterpret_cast<const uint16_t *>(&sb);
    g.s = __bfloat162float(sb);
    g.mode = (g.s == 0.0f) ? 0 : (g.s < 1.17549435e-38f ? 2 : 1);
    g.r = (g.mode == 1) ? rcp_approx(g.s) : 0.0f;
    return g;
}

// --- fast path: normal scale, straight-line, no per-element branches -------
// c = 1.5 * 2^23 + q as an fp32 (so bits(c) = 0x4B400000 + q).
__device__ __forceinline__ float code_fast(float x, float r) {
    return __fadd_rn(__fmaf_rn(x, r, kSnap), kToInt);
}

__device__ __forceinline__ void codes8_fast(const uint4 &v, float r, float (&c)[8]) {
    c[0] = code_fast(lo_f(v.x), r);
    c[1] = code_fast(hi_f(v.x), r);
    c[2] = code_fast(lo_f(v.y), r);
    c[3] = code_fast(hi_f(v.y), r);
    c[4] = code_fast(lo_f(v.z), r);
    c[5] = code_fast(hi_f(v.z), r);
    c[6] = code_fast(lo_f(v.w), r);
    c[7] = code_fast(hi_f(v.w), r);
}

// Eight codes (low bytes of the floats' bits) -> one low-nibble-first word.
__device__ __forceinline__ uint32_t pack8(const float (&c)[8]) {
    const uint32_t b0 = __float_as_uint(c[0]), b1 = __float_as_uint(c[1]);
    const uint32_t b2 = __float_as_uint(c[2]), b3 = __float_as_uint(c[3]);
    const uint32_t b4 = __float_as_uint(c[4]), b5 = __float_as_uint(c[5]);
    const uint32_t b6 = __float_as_uint(c[6]), b7 = __float_as_uint(c[7]);
    // even = bytes [q0, q2, q4, q6], odd = [q1, q3, q5, q7]
    const uint32_t even = __byte_perm(__byte_perm(b0, b2, 0x0040), __byte_perm(b4, b6, 0x0040),
                                      0x5410);
    const uint32_t odd = __byte_perm(__byte_perm(b1, b3, 0x0040), __byte_perm(b5, b7, 0x0040),
                                     0x5410);
    return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

// Eight codes -> four BF16x2 words of bf16_rne(q * s).  With
// neg_cs = -(1.5 * 2^23) * s (exact: s has 8 significant bits and 3 * s has
// at most 10, as long as s <= 2^100), fma(c, s, neg_cs) = (c - 1.5 * 2^23) * s
// = q * s exactly, rounded once to BF16 by the conversion; q == 0 gives +0.
__device__ __forceinline__ uint4 dequant8_fast(const float (&c)[8], float s, float neg_cs) {
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float v0 = __fmaf_rn(c[2 * j], s, neg_cs);
        const float v1 = __fmaf_rn(c[2 * j + 1], s, neg_cs);
        __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
        o[j] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}


// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction per two
// lanes of an IEEE fma / add, each rounded to nearest even as the scalar form).
__device__ __forceinline__ uint64_t f2_splat(float x) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
    return r;
}
// The two BF16 halves of a word, widened exactly: {low half, high half}.
__device__ __forceinline__ uint64_t f2_from_bf16x2(uint32_t w) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// Both lanes rounded to BF16 (nearest even), low lane into the low half.
__device__ __forceinline__ uint32_t f2_to_bf16x2(uint64_t d) {
    uint32_t r;
    asm("{\n\t.reg .f32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(r)
        : "l"(d));
    return r;
}

// One group of 32 BF16 values (16 words, natural order) -> the 16 BF16x2 words
// of bf16_rne(q * s), natural order; exact for every finite input.  The fast
// path needs no clamp: a normal BF16 scale is within 2^-9 of amax / 7, so
// |w / s| <= 7.03.  The slow path (zero, subnormal or huge scale) divides in
// IEEE fp32 and clamps to [-8, 7]: a subnormal scale has 1..7 significant
// bits, so there amax / s reaches 8 and more (amax bits 0x001F: s = 4 * 2^-133,
// 31/4 = 7.75 -> 7; a negative group of that size gives -8).
__device__ __forceinline__ void fake_quant_group(const uint32_t (&v)[16], uint32_t (&o)[16]) {
    const GroupScale gs = make_scale(group_amax_bits(v));
    if (gs.mode == 1 && gs.s <= 1.2676506e30f) {
        // code_fast and dequant8_fast's arithmetic, two weights per instruction
        const uint64_t r2 = f2_splat(gs.r), snap2 = f2_splat(kSnap), toint2 = f2_splat(kToInt);
        const uint64_t s2 = f2_splat(gs.s), ncs2 = f2_splat(-kMagic * gs.s);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint64_t c = f2_add(f2_fma(f2_from_bf16x2(v[j]), r2, snap2), toint2);
            o[j] = f2_to_bf16x2(f2_fma(c, s2, ncs2));
        }
    } else {
        const float s = gs.s;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float xs[2] = {lo_f(v[j]), hi_f(v[j])};
            float d[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // A subnormal s carries as few as one significant bit, so
                // |w / s| can exceed 7.5 here: the clamp to [-8, 7] fires.
                const float q = (s == 0.0f)
                                    ? 0.0f
                                    : fminf(fmaxf((float)__float2int_rn(__fdiv_rn(xs[h], s)), -8.0f), 7.0f);
                d[h] = __fmul_rn(q, s);                       // exact
            }
            __nv_bfloat162 hh = __floats2bfloat162_rn(d[0], d[1]);
            o[j] = *reinterpret_cast<uint32_t *>(&hh);
        }
    }
}

}  // namespace qdq
}  // namespace w4
