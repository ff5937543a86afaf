// w4_quant.cu -- group-32 INT4 quantizers: fake quantization (QDQ), real
// quantization + packing, the STE backward copy and the unpack/dequant helper.
//
// Method (INT4 QAT blog, fake quantization and Fig. 4; reportify.cn
// "量化感知训练" [10][11][32]; "量化基础" §2.2): per group of 32 consecutive
// BF16 weights along K, s = bf16_rne(fl32(amax / 7)),
// q = clamp(rint_half_even(w / s), -8, 7), Wdq = bf16_rne(q * s), codes packed
// low nibble first, eight per int32.
//
// Layout of the work: one thread owns one group (32 consecutive elements,
// 64 bytes read as two 32-byte loads when W is 32-byte aligned), so the amax
// needs no shuffles and the scale is formed once per group; the packed output
// is one 16-byte store per thread (consecutive across the warp).  Grid-stride
// loop with two groups (128 bytes) in flight per thread and streaming loads
// and stores: the kernels are HBM-bound, and per-element integer work is what
// limits them short of that, so it is kept to the minimum.
//
// Division-free exact arithmetic.
//  * Scale: s32 = fl32(amax / 7) is formed by quotient refinement with one FMA
//    residual step (Markstein): q0 = fl(a * c), r = fma(-q0, 7, a),
//    s32 = fma(r, c, q0), c = fl32(1/7).  This equals the IEEE quotient for
//    every finite BF16 amax (checked exhaustively on the host by
//    tests/test_kernel_arith.py).
//  * Codes: they must equal rint_half_even of the IEEE fp32 quotient
//    fl32(w / s).  With w and s both BF16 (8-bit significands) the exact
//    quotient y = w / s is either exactly a half-integer or at least 1/510 away
//    from every half-integer (write both as integer * 2^e; the numerator of
//    y - (j + 1/2) is a nonzero integer multiple of a power of two that the
//    denominator bounds), and fl32 never moves y across or onto a
//    half-integer.  The kernel forms t = w * r with r = rcp.approx(s) (relative
//    error <= 2^-23, so |t - y| < 1e-6 for |y| <= 7.03), snaps t to the 2^-10
//    grid with one fused multiply-add against 1.5 * 2^13, then rounds the
//    snapped value to an integer, ties to even, by adding the constant that
//    brings it to 1.5 * 2^23.  Snapping maps exact ties onto the half-integer
//    and keeps every other quotient strictly on its own side, so the result
//    equals rint_half_even(y).  The code is then the low byte of the float's
//    bits (bits = 0x4B400000 + q).  The fast path needs no clamp: a normal
//    BF16 scale is within 2^-9 of amax / 7, so |y| <= 7.03.  Scales below
//    2^-126 (subnormal) take the plain IEEE-division path, which clamps to
//    [-8, 7]: such a scale has 1..7 significant bits, so amax / s can round to
//    8 or more there (amax bits 0x001F give s = 4 * 2^-133 and 7.75), and a
//    negative group then gets code -8.
#include <algorithm>

#include "w4_common.cuh"
#include "w4_qdq.cuh"

namespace w4 {

namespace {

using namespace qdq;

// --- slow path: zero, subnormal or huge scale; codes by IEEE division -------
// Handles one whole 8-element item and writes its outputs (kept out of line so
// that the fast path's registers are unaffected).
template <int MODE>
__device__ __forceinline__ void item_slow(uint4 v, float s, uint32_t *Wq, uint4 *Wdq, int64_t i) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float c[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float xs[2] = {lo_f(w[j]), hi_f(w[j])};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // clamp to [-8, 7]: with a subnormal s (1..7 significant bits)
            // the quotient can round past the INT4 range
            const float q = (s == 0.0f)
                                ? 0.0f
                                : fminf(fmaxf((float)__float2int_rn(__fdiv_rn(xs[h], s)), -8.0f), 7.0f);
            c[2 * j + h] = __fadd_rn(q, kMagic);
        }
    }
    if (MODE == 0) {
        Wq[i] = pack8(c);
    } else {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float v0 = __fmul_rn(__fsub_rn(c[2 * j], kMagic), s);       // exact
            const float v1 = __fmul_rn(__fsub_rn(c[2 * j + 1], kMagic), s);
            __nv_bfloat162 hh = __floats2bfloat162_rn(v0, v1);
            o[j] = *reinterpret_cast<uint32_t *>(&hh);
        }
        Wdq[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// A whole group on the slow path, out of line so that the fast path keeps its
// registers.
template <int MODE>
__device__ __noinline__ void group_slow(uint4 c0, uint4 c1, uint4 c2, uint4 c3, float s,
                                        uint32_t *Wq, uint4 *Wdq, int64_t i0) {
    item_slow<MODE>(c0, s, Wq, Wdq, i0);
    item_slow<MODE>(c1, s, Wq, Wdq, i0 + 1);
    item_slow<MODE>(c2, s, Wq, Wdq, i0 + 2);
    item_slow<MODE>(c3, s, Wq, Wdq, i0 + 3);
}

constexpr int kUnroll = 4;
constexpr int kThreads = 256;
constexpr int kGroupsInFlight = 2;
constexpr int kQuantBlocksPerSm = 3;

// 32-byte streaming (evict-first) global load / store; 32-byte aligned address.
struct u32x8 {
    uint32_t v[8];
};

__device__ __forceinline__ u32x8 ld256_cs(const void *p) {
    u32x8 r;
    asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]), "=r"(r.v[4]),
                   "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st256_cs(void *p, const u32x8 &r) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(r.v[0]), "r"(r.v[1]), "r"(r.v[2]), "r"(r.v[3]), "r"(r.v[4]), "r"(r.v[5]),
                 "r"(r.v[6]), "r"(r.v[7])
                 : "memory");
}

// 64 bytes (one group) from global memory: two 32-byte loads (V8, 32-byte
// aligned source) or four 16-byte loads; streaming (evict-first).
template <bool V8>
__device__ __forceinline__ void load_group(const uint32_t *p, uint32_t (&v)[16]) {
    if (V8) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const u32x8 r = ld256_cs(p + 8 * h);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[8 * h + j] = r.v[j];
        }
    } else {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint4 t = __ldcs(reinterpret_cast<const uint4 *>(p) + h);
            v[4 * h] = t.x; v[4 * h + 1] = t.y; v[4 * h + 2] = t.z; v[4 * h + 3] = t.w;
        }
    }
}

template <bool V8>
__device__ __forceinline__ void store_group(uint32_t *p, const uint32_t (&v)[16]) {
    if (V8) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            u32x8 r;
#pragma unroll
            for (int j = 0; j < 8; ++j) r.v[j] = v[8 * h + j];
            st256_cs(p + 8 * h, r);
        }
    } else {
#pragma unroll
        for (int h = 0; h < 4; ++h)
            __stcs(reinterpret_cast<uint4 *>(p) + h,
                   make_uint4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]));
    }
}

// MODE 0: quantize + pack (Wq, S).  MODE 1: fake quant (Wdq, optional S).
// One thread per group of 32 weights; V8: W (and Wdq) 32-byte aligned.
template <int MODE, bool V8>
__global__ void __launch_bounds__(kThreads, kQuantBlocksPerSm) quant_kernel(const uint32_t *__restrict__ W,
                                                         uint32_t *__restrict__ Wdq,
                                                         uint32_t *__restrict__ Wq,
                                                         uint16_t *__restrict__ S,
                                                         int64_t ngroups) {
    griddep_launch_dependents();       // a GEMM after this waits for its completion
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < ngroups;
         base += kGroupsInFlight * T) {
        uint32_t v[kGroupsInFlight][16];
#pragma unroll
        for (int u = 0; u < kGroupsInFlight; ++u) {
            const int64_t g = base + u * T;
            if (g < ngroups) load_group<V8>(W + 16 * g, v[u]);
        }
#pragma unroll
        for (int u = 0; u < kGroupsInFlight; ++u) {
            const int64_t g = base + u * T;
            if (g >= ngroups) break;
            const GroupScale gs = make_scale(group_amax_bits(v[u]));
            // the fast path needs a normal scale (and, for the BF16 output, no
            // overflow of 1.5 * 2^23 * s)
            const bool fast = gs.mode == 1 && (MODE == 0 || gs.s <= 1.2676506e30f);
            if (fast) {
                if (MODE == 0) {
                    uint32_t w[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float cd[8];
                        codes8_fast(make_uint4(v[u][4 * c], v[u][4 * c + 1], v[u][4 * c + 2],
                                               v[u][4 * c + 3]),
                                    gs.r, cd);
                        w[c] = pack8(cd);
                    }
                    __stcs(reinterpret_cast<uint4 *>(Wq) + g, make_uint4(w[0], w[1], w[2], w[3]));
                } else {
                    uint32_t o[16];
                    const float neg_cs = -kMagic * gs.s;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float cd[8];
                        codes8_fast(make_uint4(v[u][4 * c], v[u][4 * c + 1], v[u][4 * c + 2],
                                               v[u][4 * c + 3]),
                                    gs.r, cd);
                        const uint4 d = dequant8_fast(cd, gs.s, neg_cs);
                        o[4 * c] = d.x; o[4 * c + 1] = d.y; o[4 * c + 2] = d.z; o[4 * c + 3] = d.w;
                    }
                    store_group<V8>(Wdq + 16 * g, o);
                }
            } else {
                group_slow<MODE>(make_uint4(v[u][0], v[u][1], v[u][2], v[u][3]),
                                 make_uint4(v[u][4], v[u][5], v[u][6], v[u][7]),
                                 make_uint4(v[u][8], v[u][9], v[u][10], v[u][11]),
                                 make_uint4(v[u][12], v[u][13], v[u][14], v[u][15]), gs.s, Wq,
                                 reinterpret_cast<uint4 *>(Wdq), 4 * g);
            }
            if (S != nullptr) S[g] = gs.bits;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 4) copy16_kernel(const uint4 *__restrict__ src,
                                                             uint4 *__restrict__ dst,
                                                             int64_t n16) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n16;
         base += kUnroll * T) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * T;
            if (i < n16) v[u] = __ldcs(src + i);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * T;
            if (i < n16) __stcs(dst + i, v[u]);
        }
    }
}

// The same copy in 32-byte units (both pointers 32-byte aligned): twice the
// bytes in flight per thread.
__global__ void __launch_bounds__(kThreads, 4) copy32_kernel(const u32x8 *__restrict__ src,
                                                             u32x8 *__restrict__ dst,
                                                             int64_t n32) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n32;
         base += kUnroll * T) {
        u32x8 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * T;
            if (i < n32) v[u] = ld256_cs(src + i);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * T;
            if (i < n32) st256_cs(dst + i, v[u]);
        }
    }
}

__global__ void copy2_tail_kernel(const uint16_t *__restrict__ src, uint16_t *__restrict__ dst,
                                  int64_t begin, int64_t n) {
    const int64_t i = begin + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = src[i];
}

// One thread = 4 words = one group of 32 codes sharing one scale.
__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint4 *__restrict__ Wq,
                                                           const uint16_t *__restrict__ S,
                                                           uint4 *__restrict__ Wdq,
                                                           int64_t ngroups) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += T) {
        const uint4 w = __ldcs(Wq + g);
        const uint32_t s2 = bf16x2_splat(S[g]);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
            dequant_word(ws[j], s2, o);
            __stcs(Wdq + 4 * g + j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

// ---- asymmetric (zero-point) groups: the affine map of the quantization
// tutorial (§2.1) with its asymmetric scale and zero point (§2.3) over the
// unsigned INT4 range [0, 15]:
//   s = bf16_rne(fl32(fl32(x_max - x_min) / 15)),
//   z = clamp(rint_even(0 - fl32(x_min / s)), 0, 15),
//   q = clamp(rint_even(fl32(x / s)) + z, 0, 15),   q = z = 0 when s == 0.
// The scale's quotient is an IEEE division (its numerator is any fp32
// difference, not a BF16 value).  The per-element quotients need none: the
// symmetric path's argument carries over with a wider range.  For a normal
// BF16 scale, |x / s| <= 256 * 15 * (1 + 2^-8) < 3856 (two distinct BF16
// values differ by at least 1/256 of the larger magnitude), and x / s is
// either exactly a half-integer or more than 1/510 away from every one
// (both operands have 8-bit significands).  So t = x * rcp.approx(s), off by
// at most 3856 * 2^-23 < 4.6e-4, snapped to the 2^-9 grid by one fused
// multiply-add against 1.5 * 2^14 (ulp 2^-9 on [2^14, 2^15)), lands on the
// half-integer exactly for a tie and stays strictly on its own side
// otherwise; adding 1.5 * 2^23 - 1.5 * 2^14 then rounds it to an integer,
// ties to even, as rint_even(fl32(x / s)) does (fl32 moves a quotient below
// 4096 by at most 2^-13, never onto or across a half-integer).  The zero point
// is the same code of x_min, negated: rint_even(-v) = -rint_even(v).  Zero,
// subnormal and huge scales (and non-finite groups) keep the IEEE divisions.

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

constexpr float kSnapZ = 24576.0f;         // 1.5 * 2^14: ulp 2^-9 around it
constexpr float kToIntZ = 12558336.0f;     // 1.5 * 2^23 - 1.5 * 2^14 (exact in fp32)

// bits(1.5 * 2^23 + rint_even(x / s)) on the fast path (|x / s| < 4096).
__device__ __forceinline__ uint32_t zp_code_bits(float x, float r) {
    return __float_as_uint(__fadd_rn(__fmaf_rn(x, r, kSnapZ), kToIntZ));
}

// One group of 32 weights (16 words, natural order) -> Wq[g] (4 words), S[g], Z[g].
__device__ __forceinline__ void quant_zp_group(const uint32_t (&v)[16], uint4 *Wq, uint16_t *S,
                                               uint8_t *Z, int64_t g) {
    uint32_t mx = v[0], mn = v[0];
#pragma unroll
    for (int j = 1; j < 16; ++j) {
        mx = bf16x2_max(mx, v[j]);
        mn = bf16x2_min(mn, v[j]);
    }
    const float xmax = fmaxf(lo_f(mx), hi_f(mx));
    const float xmin = fminf(lo_f(mn), hi_f(mn));
    const float s32 = __fdiv_rn(__fsub_rn(xmax, xmin), 15.0f);
    const __nv_bfloat16 sb = __float2bfloat16_rn(s32);
    const float s = __bfloat162float(sb);
    uint32_t words[4] = {0u, 0u, 0u, 0u};
    uint32_t z = 0u;
    if (s >= 1.17549435e-38f && s <= 1.2676506e30f) {
        const float r = rcp_approx(s);
        // z = clamp(-rint_even(x_min / s), 0, 15); codes relative to 1.5 * 2^23
        z = (uint32_t)__vimin_s32_relu((int)(0x4B400000u - zp_code_bits(xmin, r)), 15);
        const uint32_t zoff = z - 0x4B400000u;
        const uint64_t r2 = f2_splat(r), snap2 = f2_splat(kSnapZ), toint2 = f2_splat(kToIntZ);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint64_t c = f2_add(f2_fma(f2_from_bf16x2(v[j]), r2, snap2), toint2);
            const uint32_t q0 = (uint32_t)__vimin_s32_relu((int)((uint32_t)c + zoff), 15);
            const uint32_t q1 = (uint32_t)__vimin_s32_relu((int)((uint32_t)(c >> 32) + zoff), 15);
            words[j >> 2] |= (q0 | (q1 << 4)) << (8 * (j & 3));
        }
    } else if (s != 0.0f) {
        const float zf = fminf(fmaxf(rintf(__fsub_rn(0.0f, __fdiv_rn(xmin, s))), 0.0f), 15.0f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float x2[2] = {lo_f(v[j]), hi_f(v[j])};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float c = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(x2[h], s)), zf), 0.0f), 15.0f);
                const int i = 2 * j + h;               // element of the group
                words[i >> 3] |= (uint32_t)c << (4 * (i & 7));
            }
        }
        z = (uint32_t)zf;
    }
    __stcs(Wq + g, make_uint4(words[0], words[1], words[2], words[3]));
    S[g] = *reinterpret_cast<const uint16_t *>(&sb);
    Z[g] = (uint8_t)z;
}

// One thread per group of 32 weights, two groups in flight per thread.
template <bool V8>
__global__ void __launch_bounds__(kThreads, kQuantBlocksPerSm)
    quant_zp_kernel(const uint32_t *__restrict__ W, uint4 *__restrict__ Wq,
                    uint16_t *__restrict__ S, uint8_t *__restrict__ Z, int64_t ngroups) {
    griddep_launch_dependents();       // a GEMM after this waits for its completion
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < ngroups;
         base += kGroupsInFlight * T) {
        uint32_t v[kGroupsInFlight][16];
#pragma unroll
        for (int u = 0; u < kGroupsInFlight; ++u) {
            const int64_t g = base + u * T;
            if (g < ngroups) load_group<V8>(W + 16 * g, v[u]);
        }
#pragma unroll
        for (int u = 0; u < kGroupsInFlight; ++u) {
            const int64_t g = base + u * T;
            if (g >= ngroups) break;
            quant_zp_group(v[u], Wq, S, Z, g);
        }
    }
}

// One thread = one group: 4 words of unsigned codes, its scale and zero point.
__global__ void __launch_bounds__(kThreads) dequant_zp_kernel(const uint4 *__restrict__ Wq,
                                                              const uint16_t *__restrict__ S,
                                                              const uint8_t *__restrict__ Z,
                                                              uint4 *__restrict__ Wdq,
                                                              int64_t ngroups) {
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += T) {
        const uint4 w = __ldcs(Wq + g);
        const uint32_t s2 = bf16x2_splat(S[g]);
        const uint32_t zb2 = zp_bias2(Z[g]);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
            dequant_word_zp(ws[j], s2, zb2, o);
            __stcs(Wdq + 4 * g + j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// One CTA per kThreads * per_thread work items: the streaming kernels run each
// thread's loop body once (a cold 100 MB copy is ~7% faster this way than with
// one resident wave striding over the data); the grid-stride loops in the
// kernels only take over beyond the grid-size limit.
int grid_for(int64_t work_items, int per_thread) {
    const int64_t need = (work_items + (int64_t)kThreads * per_thread - 1) /
                         ((int64_t)kThreads * per_thread);
    return (int)std::max<int64_t>(1, std::min<int64_t>(need, INT32_MAX));
}

w4_status check_quant_args(const void *in, const void *out, int64_t rows, int64_t K, int group) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (rows < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (rows > 0 && K > ((int64_t)1 << 60) / rows) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(in) || !w4host::aligned16(out)) return W4_ERR_INVALID_ARG;
    return W4_OK;
}

}  // namespace
}  // namespace w4

using namespace w4;

extern "C" w4_status w4_fake_quant(const w4_bf16 *W, w4_bf16 *Wdq, w4_bf16 *S, int64_t rows,
                                   int64_t K, int group, void *stream) {
    w4_status st = check_quant_args(W, Wdq, rows, K, group);
    if (st != W4_OK) return st;
    if (S != nullptr && !w4host::aligned16(S)) return W4_ERR_INVALID_ARG;
    if ((const void *)W == (const void *)Wdq) return W4_ERR_INVALID_ARG;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    const int grid = grid_for(ngroups, kGroupsInFlight);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(W);
    uint32_t *o = reinterpret_cast<uint32_t *>(Wdq);
    uint16_t *s = reinterpret_cast<uint16_t *>(S);
    if (aligned32(W) && aligned32(Wdq))
        quant_kernel<1, true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, o, nullptr, s, ngroups);
    else
        quant_kernel<1, false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, o, nullptr, s, ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_quantize_pack(const w4_bf16 *W, int32_t *Wq, w4_bf16 *S, int64_t rows,
                                      int64_t K, int group, void *stream) {
    w4_status st = check_quant_args(W, Wq, rows, K, group);
    if (st != W4_OK) return st;
    if (!w4host::aligned16(S)) return W4_ERR_INVALID_ARG;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    const int grid = grid_for(ngroups, kGroupsInFlight);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(W);
    uint32_t *q = reinterpret_cast<uint32_t *>(Wq);
    uint16_t *s = reinterpret_cast<uint16_t *>(S);
    if (aligned32(W))
        quant_kernel<0, true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, nullptr, q, s, ngroups);
    else
        quant_kernel<0, false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, nullptr, q, s, ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_ste_backward(const w4_bf16 *dWdq, w4_bf16 *dW, int64_t n, void *stream) {
    if (n < 0 || !w4host::aligned16(dWdq) || !w4host::aligned16(dW)) return W4_ERR_INVALID_ARG;
    if ((const void *)dWdq == (const void *)dW || n == 0) return W4_OK;  // zero-copy identity
    const uint16_t *a = reinterpret_cast<const uint16_t *>(dWdq);
    uint16_t *b = reinterpret_cast<uint16_t *>(dW);
    if (a < b + n && b < a + n) return W4_ERR_INVALID_ARG;  // partial overlap
    int64_t done = 0;
    if (aligned32(a) && aligned32(b)) {
        const int64_t n32 = n / 16;
        if (n32 > 0)
            copy32_kernel<<<grid_for(n32, kUnroll), kThreads, 0, (cudaStream_t)stream>>>(
                reinterpret_cast<const u32x8 *>(a), reinterpret_cast<u32x8 *>(b), n32);
        done = n32 * 16;
    } else {
        const int64_t n16 = n / 8;
        if (n16 > 0)
            copy16_kernel<<<grid_for(n16, kUnroll), kThreads, 0, (cudaStream_t)stream>>>(
                reinterpret_cast<const uint4 *>(a), reinterpret_cast<uint4 *>(b), n16);
        done = n16 * 8;
    }
    if (done < n)
        copy2_tail_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(a, b, done, n);
    return w4host::launch_status();
}

extern "C" w4_status w4_dequant(const int32_t *Wq, const w4_bf16 *S, w4_bf16 *Wdq, int64_t rows,
                                int64_t K, int group, void *stream) {
    w4_status st = check_quant_args(Wq, Wdq, rows, K, group);
    if (st != W4_OK) return st;
    if (!w4host::aligned16(S)) return W4_ERR_INVALID_ARG;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    dequant_kernel<<<grid_for(ngroups, 1), kThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(Wq), reinterpret_cast<const uint16_t *>(S),
        reinterpret_cast<uint4 *>(Wdq), ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_quantize_pack_zp(const w4_bf16 *W, int32_t *Wq, w4_bf16 *S, uint8_t *Z,
                                         int64_t rows, int64_t K, int group, void *stream) {
    w4_status st = check_quant_args(W, Wq, rows, K, group);
    if (st != W4_OK) return st;
    if (!w4host::aligned16(S) || Z == nullptr) return W4_ERR_INVALID_ARG;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    const int grid = grid_for(ngroups, kGroupsInFlight);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(W);
    uint4 *q = reinterpret_cast<uint4 *>(Wq);
    uint16_t *s = reinterpret_cast<uint16_t *>(S);
    if (aligned32(W))
        quant_zp_kernel<true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, q, s, Z, ngroups);
    else
        quant_zp_kernel<false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, q, s, Z, ngroups);
    return w4host::launch_status();
}

extern "C" w4_status w4_dequant_zp(const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z,
                                   w4_bf16 *Wdq, int64_t rows, int64_t K, int group,
                                   void *stream) {
    w4_status st = check_quant_args(Wq, Wdq, rows, K, group);
    if (st != W4_OK) return st;
    if (!w4host::aligned16(S) || Z == nullptr) return W4_ERR_INVALID_ARG;
    const int64_t ngroups = rows * K / 32;
    if (ngroups == 0) return W4_OK;
    dequant_zp_kernel<<<grid_for(ngroups, 1), kThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(Wq), reinterpret_cast<const uint16_t *>(S), Z,
        reinterpret_cast<uint4 *>(Wdq), ngroups);
    return w4host::launch_status();
}
