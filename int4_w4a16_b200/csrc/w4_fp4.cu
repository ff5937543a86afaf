// w4_fp4.cu -- micro-scaled FP4 weight groups: real quantization + packing and
// the unpack/dequant helper (the W4A16 GEMM on FP4 codes is in w4_gemm.cu).
//
// Formats (MR-GPTQ / QuTLASS FP4 summary page: MXFP4 shares one power-of-two
// scale among 32 values, 4.25 bits per value; NVFP4 one FP8 scale among 16):
// the element is the 4-bit float E2M1 (sign, 2 exponent bits with bias 1, one
// mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).  The page fixes the
// group sizes and scale types only; the rest is read plainly:
//  * element rounding: nearest E2M1 value, ties to the even code (mantissa bit
//    0), magnitudes above 6 saturate to 6, zero is +0 (code 0);
//  * MXFP4: scale 2^e, e = floor(log2(amax)) - 2 (2 = the exponent of E2M1's
//    largest value 6), clamped to [-127, 127] and stored biased (E = e + 127)
//    in one byte (E8M0); an all-zero group stores e = 0;
//  * NVFP4: an E4M3 group scale (bias 7, largest 448) under one FP32 tensor
//    scale g = fl32(amax_tensor / (6 * 448)) (g = 1 for an all-zero tensor);
//    the group scale is amax_group / (6 g) rounded to E4M3 (nearest, ties to
//    the even code, saturating at 448); elements are rounded from w / (s g); a
//    group whose scale rounds to 0 stores zeros;
//  * dequantized value: bf16_rne(fl32(fl32(value * s) * g)) (MXFP4: g = 1;
//    value * s is exact in both formats).
// Codes are packed like the INT4 codes: eight per int32, element i of a word in
// bits [4i, 4i + 3].
//
// Where floating point decides a code, the decision is exact:
//  * MXFP4: w * 2^-e is exact in FP32 (a power-of-two scaling; only values far
//    below the first rounding threshold 0.25 can underflow), and the hardware
//    E2M1 conversion (cvt.rn.satfinite.e2m1x2.f32) rounds it to nearest even
//    with saturation; -0 codes are cleared to +0.
//  * NVFP4: both decisions take an FP32 quotient with a relative error below
//    2^-22 and round it, with the hardware conversion, scaled by 1 - 2^-b and
//    by 1 + 2^-b; when the two agree the exact quotient lies between them, so
//    that is its rounding (a tie, or any quotient within the band of a
//    rounding midpoint, gives two different codes).  Otherwise the decision is
//    taken exactly in FP64.  The group scale: amax * fl32(1 / fl32(6 g)) with
//    b = 20 through the E4M3 conversion (nearest even, saturating at 448),
//    else the IEEE FP64 quotient amax / (6 g) rounded to E4M3 from its bits.
//    An element: w * fl32(1 / fl32(s g)) with b = 19 through the E2M1
//    conversion, else |w| compared with the rounding thresholds t * s * g
//    (t in 0.25, 0.75, ..., 5), which are exact in FP64 (3 + 4 + 24
//    significant bits).  That is the same decision as rounding the quotient
//    w / (s g): an 8-bit w over a 28-bit step is either exactly a threshold or
//    at least 2^-31 relative away from it, far more than one FP64 rounding.
#include <algorithm>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two FP32 values -> one byte of E2M1 codes (a in bits 0..3, b in bits 4..7),
// nearest even with saturation at +-6.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float a, float b) {
    uint32_t d;
    asm("{.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(d)
        : "f"(a), "f"(b));
    return d;
}

// Clears the sign of every zero code (-0 -> +0) in a word of eight codes.
__device__ __forceinline__ uint32_t clear_negative_zeros(uint32_t w) {
    const uint32_t nz = ((w & 0x77777777u) + 0x77777777u) & 0x88888888u;   // bit 3: |code| != 0
    return w & (nz | 0x77777777u);
}

// ---- MXFP4 ------------------------------------------------------------------
// One thread = one group of 32 BF16 weights (64 bytes) -> 4 words + 1 scale byte.
__global__ void __launch_bounds__(kThreads) quant_mxfp4_kernel(const uint4 *__restrict__ W,
                                                               uint4 *__restrict__ Wq,
                                                               uint8_t *__restrict__ E,
                                                               int64_t ngroups) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += T) {
        uint32_t v[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 x = __ldcs(W + 4 * g + c);
            v[4 * c] = x.x;
            v[4 * c + 1] = x.y;
            v[4 * c + 2] = x.z;
            v[4 * c + 3] = x.w;
        }
        // amax of the magnitudes: BF16 bit patterns without the sign order like
        // their values (finite weights)
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t a = v[j] & 0x7FFF7FFFu;
            m = max(m, max(a & 0xFFFFu, a >> 16));
        }
        int e = 0;
        if (m != 0) {
            const int ebits = (int)((m >> 7) & 0xFFu);          // BF16 exponent field
            e = max(ebits - 129, -127);                          // floor(log2 amax) - 2
        }
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e, normal
        uint32_t words[4];
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
            uint32_t w = 0;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint32_t x = v[4 * wd + h];
                w |= e2m1x2_from_f32(__fmul_rn(bf16_lo(x), inv), __fmul_rn(bf16_hi(x), inv))
                     << (8 * h);
            }
            words[wd] = clear_negative_zeros(w);
        }
        __stcs(Wq + g, make_uint4(words[0], words[1], words[2], words[3]));
        E[g] = (uint8_t)(e + 127);
    }
}

// One thread = one group: 4 words of codes and their E8M0 scale -> 32 BF16.
__global__ void __launch_bounds__(kThreads) dequant_mxfp4_kernel(const uint4 *__restrict__ Wq,
                                                                 const uint8_t *__restrict__ E,
                                                                 uint4 *__restrict__ Wdq,
                                                                 int64_t ngroups) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += T) {
        const uint4 w = __ldcs(Wq + g);
        const float s = e8m0_to_f32(E[g]);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
            dequant_word_mxfp4(ws[j], s, o);
            __stcs(Wdq + 4 * g + j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

// ---- NVFP4 ------------------------------------------------------------------
// Tensor amax: the largest |w| as BF16 bits (sign cleared), max-reduced into
// *amax_bits (zeroed by the host first).
// W is 4-byte aligned: the pairs before its first 16-byte boundary and after
// the last whole 16 bytes are read one word at a time, the rest 16 bytes at a
// time, four loads in flight per thread.  Non-negative BF16 values order like
// their bits, so the max is a per-half unsigned max.
__global__ void __launch_bounds__(kThreads, 4) amax_bf16_kernel(const uint32_t *__restrict__ W,
                                                             int64_t n_pairs,
                                                             const uint16_t *__restrict__ tail,
                                                             unsigned int *amax_bits) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t head =
        min(n_pairs, (int64_t)(((16u - (uint32_t)(reinterpret_cast<uintptr_t>(W) & 15u)) & 15u) / 4u));
    const int64_t n16 = (n_pairs - head) / 4;
    const uint4 *W4 = reinterpret_cast<const uint4 *>(W + head);
    uint32_t m2 = 0;                                   // two running maxima, one per half
    for (int64_t base = tid; base < n16; base += 4 * T) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (base + u * T < n16) v[u] = __ldcs(W4 + base + u * T);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (base + u * T < n16) {
                m2 = __vmaxu2(m2, v[u].x & 0x7FFF7FFFu);
                m2 = __vmaxu2(m2, v[u].y & 0x7FFF7FFFu);
                m2 = __vmaxu2(m2, v[u].z & 0x7FFF7FFFu);
                m2 = __vmaxu2(m2, v[u].w & 0x7FFF7FFFu);
            }
    }
    // the unaligned head and the ragged end
    const int64_t rest = head + (n_pairs - head - 4 * n16);
    for (int64_t i = tid; i < rest; i += T) {
        const int64_t j = i < head ? i : head + 4 * n16 + (i - head);
        m2 = __vmaxu2(m2, __ldcs(W + j) & 0x7FFF7FFFu);
    }
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
    if (tail != nullptr && blockIdx.x == 0 && threadIdx.x == 0) m = max(m, (uint32_t)(*tail & 0x7FFFu));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax_bits, m);
}

// amax bits -> g = fl32(amax / 2688) in place (g = 1 when amax is 0).
__global__ void tensor_scale_kernel(unsigned int *amax_bits_to_g) {
    const float amax = __uint_as_float(*amax_bits_to_g << 16);
    float g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    if (g == 0.0f) g = 1.0f;
    *reinterpret_cast<float *>(amax_bits_to_g) = g;
}

// Nearest E4M3 code (ties to the even code, saturating at 448 = 0x7E) of v >= 0.
__device__ __forceinline__ uint32_t e4m3_code_f64(double v) {
    if (!(v > 0.0)) return 0u;
    if (v >= 448.0) return 0x7Eu;
    const long long bits = __double_as_longlong(v);
    const int e = (int)((bits >> 52) & 0x7FF) - 1023;            // floor(log2 v), v normal
    int code;
    if (e < -6) {
        code = __double2int_rn(v * 512.0);                      // subnormal grid 2^-9
    } else {
        const double mant = __longlong_as_double((bits & 0x000FFFFFFFFFFFFFll) |
                                                 0x3FF0000000000000ll);   // [1, 2)
        code = ((e + 7) << 3) + __double2int_rn((mant - 1.0) * 8.0);       // m = 8 carries
    }
    return (uint32_t)min(code, 0x7E);
}

// The E4M3 value of a code (0..0x7E) in FP64.
__device__ __forceinline__ double e4m3_value_f64(uint32_t c) {
    const int e = (int)((c >> 3) & 15u), m = (int)(c & 7u);
    return e == 0 ? (double)m * 0x1p-9 : (double)(8 + m) * ldexp(1.0, e - 10);
}

// E2M1 code of one weight from the group's step s * g (> 0): thresholds
// th[0..6] = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) * step; ties go to the even
// code, i.e. down at 0.25, 1.25, 2.5, 5 and up at 0.75, 1.75, 3.5.
__device__ __forceinline__ uint32_t e2m1_code_thresholds(float w, const double (&th)[7]) {
    const double a = fabs((double)w);
    const uint32_t c = (uint32_t)(a > th[0]) + (uint32_t)(a >= th[1]) + (uint32_t)(a > th[2]) +
                       (uint32_t)(a >= th[3]) + (uint32_t)(a > th[4]) + (uint32_t)(a >= th[5]) +
                       (uint32_t)(a > th[6]);
    return (c != 0u && w < 0.0f) ? (c | 8u) : c;
}

// The two codes of a BF16 pair (low half in bits 0..3) by the exact FP64
// thresholds of the step E4M3(sc) * g; out of line, taken rarely.
__device__ __noinline__ uint32_t e2m1_pair_exact(uint32_t x, uint32_t sc, double gd) {
    const double step = e4m3_value_f64(sc) * gd;                  // exact
    const double tq[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    double th[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) th[i] = tq[i] * step;             // exact
    return e2m1_code_thresholds(bf16_lo(x), th) | (e2m1_code_thresholds(bf16_hi(x), th) << 4);
}

// Two FP32 values -> two E4M3 codes (a in bits 0..7, b in bits 8..15), nearest
// even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(d) : "f"(a), "f"(b));
    return d;
}

// Packed pairs of FP32 (sm_100 f32x2 multiply, each lane rounded to nearest
// even as the scalar form): the two BF16 halves of a word widened exactly, a
// splat, the lane-wise product, and the lanes back.
__device__ __forceinline__ uint64_t f2_from_bf16x2_fp4(uint32_t w) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    return r;
}
__device__ __forceinline__ uint64_t f2_splat_fp4(float x) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint32_t e2m1x2_from_f2(uint64_t d) {
    uint32_t r;
    asm("{\n\t.reg .f32 lo, hi;\n\t.reg .b8 t;\n\tmov.b64 {lo, hi}, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, hi, lo;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "l"(d));
    return r;
}

constexpr int kNvPairsInFlight = 2;

// One group of 16 BF16 weights (v[0..7]) -> two words of codes; returns the
// group's E4M3 scale code.  r6g = fl32(1 / fl32(6 g)) and fast (g in
// [2^-100, 2^100]) are per tensor.
__device__ __forceinline__ uint32_t nvfp4_group(const uint32_t *v, float g, double gd, float r6g,
                                                bool fast, uint32_t *words) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = __vmaxu2(m, v[j] & 0x7FFF7FFFu);
    const float amax = __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
    uint32_t sc = 0xFFu;
    if (fast) {
        // the quotient amax / (6 g) to within 1.5 * 2^-23; both ends of the
        // 2^-20 band round alike unless it is near an E4M3 midpoint
        const float q = __fmul_rn(amax, r6g);
        const uint32_t two = e4m3x2_from_f32(__fmul_rn(q, 1.0f - 0x1p-20f), __fmul_rn(q, 1.0f + 0x1p-20f));
        if (q <= 0x1p20f && (two & 0xFFu) == (two >> 8)) sc = two & 0xFFu;
    }
    if (sc == 0xFFu) sc = e4m3_code_f64(__ddiv_rn((double)amax, 6.0 * gd));
    if (sc == 0u) {                                 // the scale rounds to 0: zeros
        words[0] = words[1] = 0u;
        return 0u;
    }
    if (fast) {
        // rs = fl32(1 / fl32(E4M3(sc) * g)) is within 2^-23 of 1 / step, so
        // w * rs is within 2^-22 of w / step; the band ends fold into rs
        const float e = e4m3_to_f32(sc);
        const float rs = __frcp_rn(__fmul_rn(e, g));
        const uint64_t lo2 = f2_splat_fp4(__fmul_rn(rs, 1.0f - 0x1p-19f));
        const uint64_t hi2 = f2_splat_fp4(__fmul_rn(rs, 1.0f + 0x1p-19f));
#pragma unroll
        for (int wd = 0; wd < 2; ++wd) {
            uint32_t w = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t x = v[4 * wd + k];
                const uint64_t x2 = f2_from_bf16x2_fp4(x);
                const uint32_t lo = e2m1x2_from_f2(f2_mul(x2, lo2));
                const uint32_t hi = e2m1x2_from_f2(f2_mul(x2, hi2));
                w |= (lo == hi ? lo : e2m1_pair_exact(x, sc, gd)) << (8 * k);
            }
            words[wd] = clear_negative_zeros(w);
        }
    } else {
#pragma unroll
        for (int wd = 0; wd < 2; ++wd) {
            uint32_t w = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) w |= e2m1_pair_exact(v[4 * wd + k], sc, gd) << (8 * k);
            words[wd] = clear_negative_zeros(w);
        }
    }
    return sc;
}

// One thread = two groups of 16 BF16 weights (64 bytes) -> 4 words + 2 scale
// bytes, two such pairs in flight.
__global__ void __launch_bounds__(kThreads) quant_nvfp4_kernel(const uint4 *__restrict__ W,
                                                               const float *__restrict__ g_dev,
                                                               uint4 *__restrict__ Wq,
                                                               uint8_t *__restrict__ S,
                                                               int64_t npairs) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    const float g = *g_dev;
    const double gd = (double)g;
    const bool fast = g >= 0x1p-100f && g <= 0x1p100f;
    const float r6g = fast ? __frcp_rn(__fmul_rn(6.0f, g)) : 0.0f;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < npairs;
         base += kNvPairsInFlight * T) {
        uint32_t v[kNvPairsInFlight][16];
#pragma unroll
        for (int u = 0; u < kNvPairsInFlight; ++u) {
            const int64_t gp = base + u * T;
            if (gp < npairs) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 x = __ldcs(W + 4 * gp + c);
                    v[u][4 * c] = x.x;
                    v[u][4 * c + 1] = x.y;
                    v[u][4 * c + 2] = x.z;
                    v[u][4 * c + 3] = x.w;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kNvPairsInFlight; ++u) {
            const int64_t gp = base + u * T;
            if (gp >= npairs) break;
            uint32_t words[4];
            const uint32_t s0 = nvfp4_group(&v[u][0], g, gd, r6g, fast, &words[0]);
            const uint32_t s1 = nvfp4_group(&v[u][8], g, gd, r6g, fast, &words[2]);
            __stcs(Wq + gp, make_uint4(words[0], words[1], words[2], words[3]));
            S[2 * gp] = (uint8_t)s0;                   // S is only byte-aligned
            S[2 * gp + 1] = (uint8_t)s1;
        }
    }
}

// One thread = 32 codes (two groups of 16) and their E4M3 scales -> 32 BF16.
__global__ void __launch_bounds__(kThreads) dequant_nvfp4_kernel(const uint4 *__restrict__ Wq,
                                                                 const uint8_t *__restrict__ S,
                                                                 float g,
                                                                 uint4 *__restrict__ Wdq,
                                                                 int64_t npairs) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t gp = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gp < npairs; gp += T) {
        const uint4 w = __ldcs(Wq + gp);
        const float s0 = e4m3_to_f32(S[2 * gp]), s1 = e4m3_to_f32(S[2 * gp + 1]);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
            dequant_word_nvfp4(ws[j], j < 2 ? s0 : s1, g, o);
            __stcs(Wdq + 4 * gp + j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

int grid_for(int64_t items) {
    const int64_t need = (items + kThreads - 1) / kThreads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(need, INT32_MAX));
}

w4_status check_fp4_args(const void *in, const void *out, const void *scales, int64_t rows,
                         int64_t K) {
    if (rows < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (rows > 0 && K > ((int64_t)1 << 60) / rows) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(in) || !w4host::aligned16(out) || scales == nullptr)
        return W4_ERR_INVALID_ARG;
    return W4_OK;
}

}  // namespace
}  // namespace w4

using namespace w4;

extern "C" w4_status w4_quantize_pack_mxfp4(const w4_bf16 *W, int32_t *Wq, uint8_t *E,
                                            int64_t rows, int64_t K, void *stream) {
    const w4_status st = check_fp4_args(W, Wq, E, rows, K);
    if (st != W4_OK) return st;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    quant_mxfp4_kernel<<<grid_for(ngroups), kThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(W), reinterpret_cast<uint4 *>(Wq), E, ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_dequant_mxfp4(const int32_t *Wq, const uint8_t *E, w4_bf16 *Wdq,
                                      int64_t rows, int64_t K, void *stream) {
    const w4_status st = check_fp4_args(Wq, Wdq, E, rows, K);
    if (st != W4_OK) return st;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    dequant_mxfp4_kernel<<<grid_for(ngroups), kThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(Wq), E, reinterpret_cast<uint4 *>(Wdq), ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_nvfp4_tensor_scale(const w4_bf16 *W, int64_t n, float *g, void *stream) {
    if (n < 0 || W == nullptr || g == nullptr || (reinterpret_cast<uintptr_t>(W) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
        return W4_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(g, 0, sizeof(float), st) != cudaSuccess) return w4host::launch_status();
    const int64_t pairs = n / 2;
    const uint16_t *tail = (n & 1) ? reinterpret_cast<const uint16_t *>(W) + (n - 1) : nullptr;
    const int grid = (int)std::min<int64_t>(std::max<int64_t>(1, (pairs + kThreads * 16 - 1) /
                                                                     (kThreads * 16)),
                                            (int64_t)w4host::num_sms() * 4);
    amax_bf16_kernel<<<grid, kThreads, 0, st>>>(reinterpret_cast<const uint32_t *>(W), pairs, tail,
                                                reinterpret_cast<unsigned int *>(g));
    tensor_scale_kernel<<<1, 1, 0, st>>>(reinterpret_cast<unsigned int *>(g));
    return w4host::launch_status();
}

extern "C" w4_status w4_quantize_pack_nvfp4(const w4_bf16 *W, const float *g, int32_t *Wq,
                                            uint8_t *S, int64_t rows, int64_t K, void *stream) {
    const w4_status st = check_fp4_args(W, Wq, S, rows, K);
    if (st != W4_OK) return st;
    if (g == nullptr || (reinterpret_cast<uintptr_t>(g) & 3u) != 0) return W4_ERR_INVALID_ARG;
    const int64_t npairs = rows * K / 32;
    if (npairs == 0) return W4_OK;
    quant_nvfp4_kernel<<<grid_for((npairs + kNvPairsInFlight - 1) / kNvPairsInFlight), kThreads, 0,
                         (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(W), g, reinterpret_cast<uint4 *>(Wq), S, npairs);
    return w4host::launch_status();
}

extern "C" w4_status w4_dequant_nvfp4(const int32_t *Wq, const uint8_t *S, float g, w4_bf16 *Wdq,
                                      int64_t rows, int64_t K, void *stream) {
    const w4_status st = check_fp4_args(Wq, Wdq, S, rows, K);
    if (st != W4_OK) return st;
    const int64_t npairs = rows * K / 32;
    if (npairs == 0) return W4_OK;
    dequant_nvfp4_kernel<<<grid_for(npairs), kThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(Wq), S, g, reinterpret_cast<uint4 *>(Wdq), npairs);
    return w4host::launch_status();
}
