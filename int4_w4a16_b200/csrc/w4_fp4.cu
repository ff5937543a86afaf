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
//  * NVFP4: the group scale is the IEEE FP64 quotient amax / (6 g) rounded to
//    E4M3 from its bits; an element's code is the hardware E2M1 rounding of
//    w * fl32(1 / (s g)) when the rounding of that FP32 quotient scaled by
//    1 - 2^-19 and by 1 + 2^-19 agree (the quotient is then at least that far
//    from every rounding midpoint, and its error is below 2^-22); otherwise
//    |w| is compared with the rounding thresholds t * s * g (t in 0.25, 0.75,
//    ..., 5), which are exact in FP64 (3 + 4 + 24 significant bits).  That is
//    the same decision as rounding the quotient w / (s g): an 8-bit w over a
//    28-bit step is either exactly a threshold or at least 2^-31 relative away
//    from it, far more than one FP64 rounding.
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
__global__ void __launch_bounds__(kThreads) amax_bf16_kernel(const uint32_t *__restrict__ W,
                                                             int64_t n_pairs,
                                                             const uint16_t *__restrict__ tail,
                                                             unsigned int *amax_bits) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs; i += T) {
        const uint32_t a = __ldcs(W + i) & 0x7FFF7FFFu;
        m = max(m, max(a & 0xFFFFu, a >> 16));
    }
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

// One thread = two groups of 16 BF16 weights (64 bytes) -> 4 words + 2 scale bytes.
__global__ void __launch_bounds__(kThreads) quant_nvfp4_kernel(const uint4 *__restrict__ W,
                                                               const float *__restrict__ g_dev,
                                                               uint4 *__restrict__ Wq,
                                                               uint8_t *__restrict__ S,
                                                               int64_t npairs) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    const float g = *g_dev;
    const double gd = (double)g;
    const double six_g = 6.0 * gd;
    for (int64_t gp = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gp < npairs; gp += T) {
        uint32_t v[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 x = __ldcs(W + 4 * gp + c);
            v[4 * c] = x.x;
            v[4 * c + 1] = x.y;
            v[4 * c + 2] = x.z;
            v[4 * c + 3] = x.w;
        }
        uint32_t words[4];
        uint32_t sc2 = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {                    // group h: v[8h .. 8h + 7]
            uint32_t m = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t a = v[8 * h + j] & 0x7FFF7FFFu;
                m = max(m, max(a & 0xFFFFu, a >> 16));
            }
            const double amax = (double)__uint_as_float(m << 16);
            const uint32_t sc = e4m3_code_f64(__ddiv_rn(amax, six_g));
            sc2 |= sc << (8 * h);
            const double step = e4m3_value_f64(sc) * gd;          // exact
            double th[7];
            const double tq[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
#pragma unroll
            for (int i = 0; i < 7; ++i) th[i] = tq[i] * step;   // exact
            // Fast path: r = w * fl32(1 / step) in FP32 is within 2^-22 of w /
            // step (relative); rounding r * (1 -+ 2^-19) with the hardware E2M1
            // conversion gives the same code at both ends unless the exact
            // quotient is within that band of a rounding midpoint (a tie
            // included), and then it is the code of the exact quotient.  Pairs
            // whose two ends differ take the exact FP64 thresholds.
            const bool fast = step > 0x1p-100;
            const float rs = fast ? (float)(1.0 / step) : 0.0f;
            constexpr float kLo = 1.0f - 0x1p-19f, kHi = 1.0f + 0x1p-19f;
#pragma unroll
            for (int wd = 0; wd < 2; ++wd) {
                uint32_t w = 0;
                if (step > 0.0) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t x = v[8 * h + 4 * wd + k];
                        const float a = bf16_lo(x), b = bf16_hi(x);
                        uint32_t byte;
                        bool exact = !fast;
                        if (fast) {
                            const float ra = __fmul_rn(a, rs), rb = __fmul_rn(b, rs);
                            const uint32_t lo = e2m1x2_from_f32(__fmul_rn(ra, kLo), __fmul_rn(rb, kLo));
                            const uint32_t hi = e2m1x2_from_f32(__fmul_rn(ra, kHi), __fmul_rn(rb, kHi));
                            byte = lo;
                            exact = lo != hi;
                        }
                        if (exact)
                            byte = e2m1_code_thresholds(a, th) | (e2m1_code_thresholds(b, th) << 4);
                        w |= byte << (8 * k);
                    }
                }
                words[2 * h + wd] = clear_negative_zeros(w);
            }
        }
        __stcs(Wq + gp, make_uint4(words[0], words[1], words[2], words[3]));
        S[2 * gp] = (uint8_t)(sc2 & 0xFFu);
        S[2 * gp + 1] = (uint8_t)(sc2 >> 8);
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
    const int grid = (int)std::min<int64_t>(std::max<int64_t>(1, (pairs + kThreads * 8 - 1) /
                                                                     (kThreads * 8)),
                                            (int64_t)w4host::num_sms() * 8);
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
    quant_nvfp4_kernel<<<grid_for(npairs), kThreads, 0, (cudaStream_t)stream>>>(
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
