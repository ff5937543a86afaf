// w4_gemv.cu -- decode-shaped W4A16 GEMM (1..8 activation rows) on the
// warp-level MMA path.
//
// What it computes (INT4 QAT blog, Fig. 4 and "zero-overhead unpacking";
// reportify.cn "量化感知训练" [32][35]):  Y[m, n] = sum_k X[m, k] * dq(W)[n, k],
// dq(W)[n, k] = bf16_rne(q[n, k] * S[n, k/32]) (or bf16_rne((q - z) * s) for
// zero-point groups, or the dequantized MXFP4 / NVFP4 value for E2M1 codes with
// scale bytes, MR-GPTQ / QuTLASS FP4 summary), FP32 accumulation, one BF16
// rounding of the result -- the product of w4_gemm.cu, for activation heights
// where streaming the packed weights from HBM, not the math, sets the time.
//
// Design (B200-first):
//  * one CTA per SM owns a contiguous range of output rows, cut at 4-row
//    granularity so that every SM streams the same number of bytes (83-84 rows
//    of 12288), and all of K for them: no partial sum leaves the SM and no
//    workspace or second kernel is needed;
//  * the rows stream as 16-row tiles x 4096 K (36 KB with their scales), one
//    TMA box per operand (a CTA's last, partial tile as 4-row boxes, so no byte
//    is fetched twice), through a ring of four shared-memory stages: enough
//    bytes in flight for HBM, few enough that the first tile lands early.  The
//    last warp done with a slot refills it, so no warp is spent on loads;
//  * 16 warps split K: warp w owns 256 of every 4096 K and keeps that slice of
//    the activations in registers as MMA B fragments;
//  * per tile a lane reads its four packed words of a row with one 16-byte
//    shared load (conflict-free: a quarter warp reads two rows' 64 contiguous
//    bytes), unpacks the codes in registers (one LOP3 per code pair and two
//    packed BF16 operations, exact: bf16_rne(q * s), the dequantized weight as
//    defined) straight into A fragments and issues mma.sync m16n8k16 (BF16 in,
//    FP32 accumulate), swap-AB: weight rows are the MMA's M, tokens its N;
//  * a warp's sums of a tile go to shared memory when the tile is done (four
//    floats per lane): the tile loop is not unrolled over the tiles, so the
//    code stays small enough for the instruction cache; at the end the 16
//    partial sums of each output are added in a fixed warp order
//    (deterministic), rounded once and stored.
// Lane (g, t) owns packed words 4t .. 4t+3 of a row's chunk, i.e. scale group t
// of the chunk and K = 128c + 32t + 8j + (0..7) for word j, for rows g and
// g + 8 of a tile.  Inside an MMA the K order follows the packed word (codes j
// and j + 4 share a register) and the activation fragments are built in the
// same order; the K sum does not depend on the order of its terms.
// Every mbarrier wait is bounded (w4_common.cuh); a timed-out CTA records the
// device status, lets its issued copies land and exits.
#include <algorithm>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kDecWarps = 16;                            // all warps compute
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kChunkK = 128;                             // 16 packed words = 4 groups
constexpr int kWarpChunks = 2;                           // chunks of one warp per K pass
constexpr int kPassChunks = kDecWarps * kWarpChunks;     // 32 chunks = 4096 K per pass
constexpr int kMaxTiles = 6;                             // 16-row tiles per CTA
constexpr int kMaxQuads = 4 * kMaxTiles;                 // 4-row units per CTA
constexpr int kNStage = 4;
constexpr int kMaxM = 8;

// Weight formats of the kernel: INT4 codes with BF16 scales (symmetric, or
// with a zero-point byte per group), or FP4 (E2M1) codes with one scale byte
// per 32 (MXFP4, E8M0) or per 16 (NVFP4, E4M3) codes.
enum : int { kFmtInt4 = 0, kFmtInt4Zp = 1, kFmtMxfp4 = 2, kFmtNvfp4 = 3 };
__host__ __device__ constexpr bool fmt_has_s(int f) { return f <= kFmtInt4Zp; }   // BF16 scales
__host__ __device__ constexpr bool fmt_has_z(int f) { return f >= kFmtInt4Zp; }   // byte box
__host__ __device__ constexpr bool fmt_fp4(int f) { return f >= kFmtMxfp4; }
// bytes of the byte box per row and 512-K block: zero points or E8M0 scales
// (one per 32 codes), E4M3 scales (one per 16)
__host__ __device__ constexpr int fmt_zbytes(int f) { return f == kFmtNvfp4 ? 32 : 16; }

template <int F>
struct DecCfg {
    // a stage as its TMA boxes land (a 16-row tile: one box per operand; a
    // partial tile: one 4-row box per 4-row unit, QW / QS / QZ apart)
    static constexpr int ZB = fmt_zbytes(F);
    static constexpr int QW = kPassChunks * 4 * 64;               // words [chunk][4 rows][16]
    static constexpr int QS = fmt_has_s(F) ? (kPassChunks / 2) * 4 * 16 : 0;  // [256 K][4][8]
    static constexpr int QZ = fmt_has_z(F) ? (kPassChunks / 4) * 4 * ZB : 0;  // [512 K][4][ZB]
    static constexpr int SOFF = 4 * QW;                           // 32 KB of words first
    static constexpr int ZOFF = 4 * (QW + QS);
    static constexpr int STAGE = 4 * (QW + QS + QZ);
    static constexpr int RING = kNStage * STAGE;
    // partial sums [warp][tile][lane][4 floats]
    static constexpr int RED_BYTES = kDecWarps * kMaxTiles * 32 * 16;
    static constexpr int SMEM = 1024 + RING + RED_BYTES;
    static_assert(QW % 1024 == 0 && QS % 512 == 0 && QZ % 512 == 0 && STAGE % 1024 == 0,
                  "box alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct DecParams {
    const uint16_t *X;    // [M, K] BF16
    uint16_t *Y;          // [M, N] BF16
    float g;              // NVFP4 tensor scale
    int M, N, K;
    int n_quads, ctas;    // 4-row units of N, CTAs they are cut over
    int kc, passes;       // K / 128 chunks, passes of 4096 K
};

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void sts128f(uint32_t addr, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ldg128_nc(const uint16_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_cta(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "r"(addr), "r"(v)
                 : "memory");
    return old;
}

// D += A * B, m16n8k16, BF16 operands, FP32 accumulators.
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Warp-uniform bounded wait.
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    const bool ok = mbar_wait(bar, parity, abort_flag);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Wait on the way out (ignores the abort flag): lets issued copies land.
__device__ __forceinline__ void dec_drain(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1; !mbar_try_wait(bar, parity); ++n) {
        if (n % kPollsPerCheck == 0 && globaltimer_ns() - t0 > kWaitLimitNs / 4) {
            record_timeout();
            return;
        }
    }
}

// Shared-memory offsets of one lane for the chunk ch of a stage.  A full tile
// is one box per operand: words [chunk][16 rows][64 B], scales [256-K block]
// [16 rows][16 B], bytes [512-K block][16 rows][ZB B]; a partial tile holds
// 4-row boxes ([chunk][4 rows][64 B], [block][4 rows][16 B], [block][4 rows]
// [ZB B]) QW / QS / QZ apart.  Row g + 8 sits a fixed distance after row g.
// The lane's byte (or, for NVFP4, its two bytes) of its group of 32 codes
// sits at group index (ch & 3) * 4 + t of the row's 512-K block.
template <int F>
struct LaneOff {
    uint32_t w, s, z;       // row g: its 16 bytes of words, its scale, its byte(s)
    uint32_t dw, ds, dz;    // row g + 8 minus row g
    __device__ __forceinline__ LaneOff(bool full, int ch, int g, int t) {
        using C = DecCfg<F>;
        constexpr int ZB = C::ZB;
        const uint32_t su = (uint32_t)(((ch & 1) * 4 + t) * 2);
        const uint32_t zu = (uint32_t)(((ch & 3) * 4 + t) * (ZB / 16));
        if (full) {
            w = (uint32_t)(ch * 1024 + g * 64 + t * 16);
            s = (uint32_t)(C::SOFF + (ch >> 1) * 256 + g * 16) + su;
            z = (uint32_t)(C::ZOFF + (ch >> 2) * 16 * ZB + g * ZB) + zu;
            dw = 512u;
            ds = 128u;
            dz = 8u * ZB;
        } else {
            w = (uint32_t)((g >> 2) * C::QW + ch * 256 + (g & 3) * 64 + t * 16);
            s = (uint32_t)(C::SOFF + (g >> 2) * C::QS + (ch >> 1) * 64 + (g & 3) * 16) + su;
            z = (uint32_t)(C::ZOFF + (g >> 2) * C::QZ + (ch >> 2) * 4 * ZB + (g & 3) * ZB) + zu;
            dw = 2u * C::QW;
            ds = 2u * C::QS;
            dz = 2u * C::QZ;
        }
    }
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}

// One word pair (rows g and g + 8) of step j into the accumulators.
template <int F, bool HI>
__device__ __forceinline__ void dec_word(uint32_t wg, uint32_t wh, uint32_t s2g, uint32_t s2h,
                                         uint32_t zg, uint32_t zh, const uint4 &x, float (&d)[4]) {
    uint32_t pg[4], ph[4] = {0u, 0u, 0u, 0u};
    if (F == kFmtInt4Zp) {
        dequant_word_k8perm_zp(wg, s2g, zp_bias2(zg), pg);
        if (HI) dequant_word_k8perm_zp(wh, s2h, zp_bias2(zh), ph);
    } else {
        dequant_word_k8perm(wg, s2g, pg);
        if (HI) dequant_word_k8perm(wh, s2h, ph);
    }
    mma_bf16_m16n8k16(d, pg[0], ph[0], pg[1], ph[1], x.x, x.y);
    mma_bf16_m16n8k16(d, pg[2], ph[2], pg[3], ph[3], x.z, x.w);
}

// FP4: one word pair with the group scales as FP32 (sg, sh) into the
// accumulators; the codes come out in natural order (codes 2j, 2j + 1 in one
// register), so these activations are not permuted.
template <int F, bool HI>
__device__ __forceinline__ void dec_word_fp4(uint32_t wg, uint32_t wh, float sg, float sh, float g,
                                             const uint4 &x, float (&d)[4]) {
    uint32_t pg[4], ph[4] = {0u, 0u, 0u, 0u};
    if (F == kFmtMxfp4) {
        dequant_word_mxfp4(wg, sg, pg);
        if (HI) dequant_word_mxfp4(wh, sh, ph);
    } else {
        dequant_word_nvfp4(wg, sg, g, pg);
        if (HI) dequant_word_nvfp4(wh, sh, g, ph);
    }
    mma_bf16_m16n8k16(d, pg[0], ph[0], pg[1], ph[1], x.x, x.y);
    mma_bf16_m16n8k16(d, pg[2], ph[2], pg[3], ph[3], x.z, x.w);
}

// One chunk of a tile, rows g and (HI) g + 8: loads, then the four words, the
// even ones into acc and the odd ones into acc2 (two independent MMA chains).
template <int F, bool HI>
__device__ __forceinline__ void dec_chunk(uint32_t slot, const LaneOff<F> &o, const uint4 (&x)[4],
                                          float g, float (&acc)[4], float (&acc2)[4]) {
    const uint4 wg = lds128(slot + o.w);
    uint4 wh = make_uint4(0u, 0u, 0u, 0u);
    if (HI) wh = lds128(slot + o.w + o.dw);
    if constexpr (fmt_fp4(F)) {
        // MXFP4: one E8M0 byte for the chunk's 32 codes; NVFP4: two E4M3
        // bytes, words 0-1 and words 2-3
        float sg0, sg1, sh0 = 0.f, sh1 = 0.f;
        if (F == kFmtMxfp4) {
            sg0 = sg1 = e8m0_to_f32(lds_u8(slot + o.z));
            if (HI) sh0 = sh1 = e8m0_to_f32(lds_u8(slot + o.z + o.dz));
        } else {
            const uint32_t zg = lds_u16(slot + o.z);
            sg0 = e4m3_to_f32(zg & 0xFFu);
            sg1 = e4m3_to_f32(zg >> 8);
            if (HI) {
                const uint32_t zh = lds_u16(slot + o.z + o.dz);
                sh0 = e4m3_to_f32(zh & 0xFFu);
                sh1 = e4m3_to_f32(zh >> 8);
            }
        }
        dec_word_fp4<F, HI>(wg.x, wh.x, sg0, sh0, g, x[0], acc);
        dec_word_fp4<F, HI>(wg.y, wh.y, sg0, sh0, g, x[1], acc2);
        dec_word_fp4<F, HI>(wg.z, wh.z, sg1, sh1, g, x[2], acc);
        dec_word_fp4<F, HI>(wg.w, wh.w, sg1, sh1, g, x[3], acc2);
    } else {
        const uint32_t sg = lds_u16(slot + o.s);
        const uint32_t zg = (F == kFmtInt4Zp) ? lds_u8(slot + o.z) : 0u;
        uint32_t sh = 0u, zh = 0u;
        if (HI) {
            sh = lds_u16(slot + o.s + o.ds);
            if (F == kFmtInt4Zp) zh = lds_u8(slot + o.z + o.dz);
        }
        const uint32_t s2g = sg | (sg << 16), s2h = sh | (sh << 16);
        dec_word<F, HI>(wg.x, wh.x, s2g, s2h, zg, zh, x[0], acc);
        dec_word<F, HI>(wg.y, wh.y, s2g, s2h, zg, zh, x[1], acc2);
        dec_word<F, HI>(wg.z, wh.z, s2g, s2h, zg, zh, x[2], acc);
        dec_word<F, HI>(wg.w, wh.w, s2g, s2h, zg, zh, x[3], acc2);
    }
}

// Stage s = (pass s / ntiles, tile s % ntiles) into slot s % kNStage; out of
// line so that the compute loop keeps its registers.
template <int F>
__device__ __noinline__ void dec_issue(const CUtensorMap *tw, const CUtensorMap *ts,
                                       const CUtensorMap *tz, const CUtensorMap *tw4,
                                       const CUtensorMap *ts4, const CUtensorMap *tz4,
                                       uint32_t bars, uint32_t base, int row0, int cta_quads,
                                       int ntiles, int *issued, int s) {
    using C = DecCfg<F>;
    const int slot = s % kNStage, pass = s / ntiles, tile = s % ntiles;
    const int nq = min(4, cta_quads - 4 * tile);
    const uint32_t fb = bars + (uint32_t)(slot * 8);
    const uint32_t dst = base + (uint32_t)(slot * C::STAGE);
    const int r = row0 + 16 * tile;
    atomicMax(issued, s + 1);
    mbar_arrive_expect_tx(fb, (uint32_t)(nq * (C::QW + C::QS + C::QZ)));
    if (nq == 4) {
        tma_load_3d(dst, tw, fb, 0, r, pass * kPassChunks);
        if (fmt_has_s(F)) tma_load_3d(dst + C::SOFF, ts, fb, 0, r, pass * (kPassChunks / 2));
        if (fmt_has_z(F)) tma_load_3d(dst + C::ZOFF, tz, fb, 0, r, pass * (kPassChunks / 4));
    } else {
        for (int q = 0; q < nq; ++q) {
            tma_load_3d(dst + q * C::QW, tw4, fb, 0, r + 4 * q, pass * kPassChunks);
            if (fmt_has_s(F))
                tma_load_3d(dst + C::SOFF + q * C::QS, ts4, fb, 0, r + 4 * q,
                            pass * (kPassChunks / 2));
            if (fmt_has_z(F))
                tma_load_3d(dst + C::ZOFF + q * C::QZ, tz4, fb, 0, r + 4 * q,
                            pass * (kPassChunks / 4));
        }
    }
}

template <int F>
__global__ void __launch_bounds__(kDecThreads, 1)
    w4a16_dec_kernel(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap ts,
                     const __grid_constant__ CUtensorMap tz, const __grid_constant__ CUtensorMap tw4,
                     const __grid_constant__ CUtensorMap ts4, const __grid_constant__ CUtensorMap tz4,
                     const DecParams p) {
    using C = DecCfg<F>;
    extern __shared__ __align__(1024) uint8_t dec_smem[];
    __shared__ __align__(8) uint64_t full_bar[kNStage];     // stage landed (TMA bytes)
    __shared__ uint32_t slot_done[kNStage];                 // warps done with a slot (grows)
    __shared__ int abort_flag;
    __shared__ int issued;                                   // stages whose loads were issued

    const uint32_t raw = smem_u32(dec_smem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t red = base + (uint32_t)C::RING;          // partial sums
    const float *redf = reinterpret_cast<const float *>(dec_smem + (red - raw));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int q0 = (int)((int64_t)blockIdx.x * p.n_quads / p.ctas);
    const int q1 = (int)((int64_t)(blockIdx.x + 1) * p.n_quads / p.ctas);
    const int cta_quads = q1 - q0;
    const int row0 = 4 * q0;
    const int cta_rows = min(p.N, 4 * q1) - row0;
    const int ntiles = (cta_quads + 3) / 4;
    const int nstages = ntiles * p.passes;

    // this warp's two chunks of the activations in B-fragment order (tokens >=
    // M and K beyond the end are zero): lane (g, t) holds token g's
    // K = 128c + 32t + 8j + (0..7).  Pass 0's requests go out ahead of the
    // first weight stages.
    uint4 xr[kWarpChunks][4];
    int na = 0;
    auto load_x = [&](int pass) {
        const int c_first = pass * kPassChunks + warp * kWarpChunks;
        na = max(0, min(kWarpChunks, p.kc - c_first));
#pragma unroll
        for (int cl = 0; cl < kWarpChunks; ++cl)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                xr[cl][j] = make_uint4(0u, 0u, 0u, 0u);
                if (cl < na && g < p.M)
                    xr[cl][j] = ldg128_nc(p.X + (size_t)g * p.K +
                                          (size_t)(c_first + cl) * kChunkK + 32 * t + 8 * j);
            }
    };
#define DEC_ISSUE(s_)                                                                        \
    dec_issue<F>(&tw, &ts, &tz, &tw4, &ts4, &tz4, smem_u32(&full_bar[0]), base, row0, cta_quads, \
                  ntiles, &issued, (s_))
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tw);
        if (fmt_has_s(F)) tma_prefetch_desc(&ts);
        if (fmt_has_z(F)) tma_prefetch_desc(&tz);
        for (int i = 0; i < kNStage; ++i) {
            mbar_init(smem_u32(&full_bar[i]), 1u);
            slot_done[i] = 0u;
        }
        abort_flag = 0;
        issued = 0;
        fence_mbar_init();
    }
    // the kernel before this one on the stream may still be running: its
    // outputs (X among them) are read only after it completes
    griddep_wait();
    griddep_launch_dependents();
    load_x(0);
    if (threadIdx.x == 0)
        for (int s = 0; s < min(nstages, kNStage); ++s) DEC_ISSUE(s);
    __syncthreads();

    bool ok = true;
    for (int pass = 0; pass < p.passes && ok; ++pass) {
        if (pass > 0) load_x(pass);
        uint4 xf[kWarpChunks][4];
#pragma unroll
        for (int cl = 0; cl < kWarpChunks; ++cl)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xf[cl][j] = fmt_fp4(F) ? xr[cl][j] : permute_chunk8(xr[cl][j]);
        for (int i = 0; i < ntiles; ++i) {
            const int s = pass * ntiles + i;
            const int slot = s % kNStage;
            if (!dec_wait(smem_u32(&full_bar[slot]), (uint32_t)((s / kNStage) & 1), &abort_flag)) {
                ok = false;
                break;
            }
            const int nq = min(4, cta_quads - 4 * i);
            const bool full = nq == 4, hi_rows = nq > 2;       // rows 8..15 of the tile
            const uint32_t sb = base + (uint32_t)(slot * C::STAGE);
            float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cl = 0; cl < kWarpChunks; ++cl) {
                if (cl < na) {
                    const LaneOff<F> o(full, warp * kWarpChunks + cl, g, t);
                    if (hi_rows)
                        dec_chunk<F, true>(sb, o, xf[cl], p.g, acc, acc2);
                    else
                        dec_chunk<F, false>(sb, o, xf[cl], p.g, acc, acc2);
                }
            }
            // This warp's shared-memory reads of the slot are complete; the last
            // warp done with it (the counter only grows: 16 arrivals per use)
            // refills it with stage s + kNStage.
            __syncwarp();
            if (lane == 0 && s + kNStage < nstages) {
                const uint32_t before = atom_add_acq_rel_cta(smem_u32(&slot_done[slot]), 1u);
                if (before == (uint32_t)(kDecWarps * (s / kNStage + 1) - 1) && !abort_flag)
                    DEC_ISSUE(s + kNStage);
            }
            // the tile's sums into this warp's partial sums
            const uint32_t ra = red + (uint32_t)(((warp * kMaxTiles + i) * 32 + lane) * 16);
            float4 v = make_float4(acc[0] + acc2[0], acc[1] + acc2[1], acc[2] + acc2[2],
                                   acc[3] + acc2[3]);
            if (pass > 0) {
                const float4 prev = lds128f(ra);
                v = make_float4(prev.x + v.x, prev.y + v.y, prev.z + v.z, prev.w + v.w);
            }
            sts128f(ra, v);
        }
    }
#undef DEC_ISSUE
    // ---- every warp's partial sums are in shared memory: add them in warp
    // order for each output (row r of the CTA, token m)
    __syncthreads();
    if (!abort_flag) {
        const int items = cta_rows * p.M;
        for (int it = threadIdx.x; it < items; it += kDecThreads) {
            const int m = it / cta_rows, r = it - m * cta_rows;
            const int tile = r >> 4, rr = r & 15;
            const int ln = (rr & 7) * 4 + (m >> 1), el = (rr >> 3) * 2 + (m & 1);
            const float *src = redf + ((size_t)tile * 32 + ln) * 4 + el;
            float sum = src[0];
#pragma unroll
            for (int w = 1; w < kDecWarps; ++w) sum += src[(size_t)w * kMaxTiles * 32 * 4];
            const __nv_bfloat16 b = __float2bfloat16_rn(sum);
            p.Y[(size_t)m * p.N + row0 + r] = *reinterpret_cast<const uint16_t *>(&b);
        }
    }
    // after a timeout: every issued copy lands before the shared memory goes away
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag) {
        for (int s = max(0, issued - kNStage); s < issued; ++s)
            dec_drain(smem_u32(&full_bar[s % kNStage]), (uint32_t)((s / kNStage) & 1));
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int F>
w4_status dec_launch(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z,
                     float g, w4_bf16 *Y, int M, int N, int K, cudaStream_t stream) {
    using C = DecCfg<F>;
    const int sms = w4host::num_sms();
    DecParams p = {};
    p.X = reinterpret_cast<const uint16_t *>(X);
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.g = g;
    p.M = M;
    p.N = N;
    p.K = K;
    p.n_quads = (N + 3) / 4;
    // one CTA per SM, more CTAs only when an SM's share would exceed the rows
    // whose partial sums one CTA holds
    p.ctas = std::max(std::min(sms, p.n_quads), (p.n_quads + kMaxQuads - 1) / kMaxQuads);
    p.kc = K / kChunkK;
    p.passes = (p.kc + kPassChunks - 1) / kPassChunks;
    const int max_quads = (p.n_quads + p.ctas - 1) / p.ctas;
    if (max_quads > kMaxQuads) return W4_ERR_UNSUPPORTED;
    const size_t smem = (size_t)C::SMEM;

    // packed words as [K / 128 chunks][N rows][16 words],
    // BF16 scales as [K / 256 blocks][N rows][8 groups], zero points or FP4
    // scale bytes as [K / 512 blocks][N rows][16 or 32 bytes]: 16-row boxes for
    // whole tiles, 4-row boxes for a CTA's partial last tile
    CUtensorMap tw, ts, tz, tw4, ts4, tz4;
    for (int rows : {16, 4}) {
        CUtensorMap *mw = rows == 16 ? &tw : &tw4, *ms = rows == 16 ? &ts : &ts4;
        CUtensorMap *mz = rows == 16 ? &tz : &tz4;
        {
            cuuint64_t dims[3] = {16u, (cuuint64_t)N, (cuuint64_t)(K / kChunkK)};
            cuuint64_t strides[2] = {(cuuint64_t)K / 2, 64u};
            cuuint32_t box[3] = {16u, (cuuint32_t)rows, (cuuint32_t)kPassChunks};
            if (w4host::encode_tiled(mw, CU_TENSOR_MAP_DATA_TYPE_INT32, 3,
                                     const_cast<int32_t *>(Wq), dims, strides, box,
                                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
                return W4_ERR_CUDA;
        }
        if (fmt_has_s(F)) {
            cuuint64_t dims[3] = {8u, (cuuint64_t)N, (cuuint64_t)(K / 256)};
            cuuint64_t strides[2] = {(cuuint64_t)K / 16, 16u};
            cuuint32_t box[3] = {8u, (cuuint32_t)rows, (cuuint32_t)(kPassChunks / 2)};
            if (w4host::encode_tiled(ms, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                                     const_cast<w4_bf16 *>(S), dims, strides, box,
                                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
                return W4_ERR_CUDA;
        }
        if (fmt_has_z(F)) {
            constexpr int ZB = C::ZB;
            cuuint64_t dims[3] = {(cuuint64_t)ZB, (cuuint64_t)N, (cuuint64_t)(K / 512)};
            cuuint64_t strides[2] = {(cuuint64_t)K / 512 * ZB, (cuuint64_t)ZB};
            cuuint32_t box[3] = {(cuuint32_t)ZB, (cuuint32_t)rows, (cuuint32_t)(kPassChunks / 4)};
            if (w4host::encode_tiled(mz, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(Z),
                                     dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
                return W4_ERR_CUDA;
        }
        if (!fmt_has_s(F)) *ms = *mz;                // not read
        if (!fmt_has_z(F)) *mz = *ms;                // not read
    }
    auto kern = w4a16_dec_kernel<F>;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return w4host::launch_status();
        configured = true;
    }
    const cudaError_t e = w4host::launch_pdl(kern, dim3(p.ctas), dim3(kDecThreads), (size_t)smem,
                                             stream, tw, ts, tz, tw4, ts4, tz4, p);
    if (e != cudaSuccess) {
        w4host::set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    return w4host::launch_status();
}

}  // namespace
}  // namespace w4

// Shapes the warp-level MMA path takes: 1..8 activation rows (from 9 rows on,
// the tensor-memory kernel), K a multiple of 256 (whole 256-wide scale blocks
// per TMA box).
bool w4host::gemv_supported(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && M <= w4::kMaxM && N >= 1 && N <= (1 << 30) && K >= 256 && (K % 256) == 0 &&
           K <= (1 << 24);
}

w4_status w4host::gemv_launch(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, w4_bf16 *Y,
                              int64_t M, int64_t N, int64_t K, void *stream) {
    if (!gemv_supported(M, N, K)) return W4_ERR_UNSUPPORTED;
    return w4::dec_launch<w4::kFmtInt4>(X, Wq, S, nullptr, 1.0f, Y, (int)M, (int)N, (int)K,
                                        (cudaStream_t)stream);
}

w4_status w4host::gemv_launch_zp(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                                 const uint8_t *Z, w4_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                 void *stream) {
    if (!gemv_supported(M, N, K) || (K % 512) != 0 || !aligned16(Z)) return W4_ERR_UNSUPPORTED;
    return w4::dec_launch<w4::kFmtInt4Zp>(X, Wq, S, Z, 1.0f, Y, (int)M, (int)N, (int)K,
                                          (cudaStream_t)stream);
}

w4_status w4host::gemv_launch_fp4(int fp4, const w4_bf16 *X, const int32_t *Wq, const uint8_t *SB,
                                  float g, w4_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                  void *stream) {
    if (!gemv_supported(M, N, K) || (K % 512) != 0 || !aligned16(SB)) return W4_ERR_UNSUPPORTED;
    if (fp4 == 1)
        return w4::dec_launch<w4::kFmtMxfp4>(X, Wq, nullptr, SB, 1.0f, Y, (int)M, (int)N, (int)K,
                                             (cudaStream_t)stream);
    return w4::dec_launch<w4::kFmtNvfp4>(X, Wq, nullptr, SB, g, Y, (int)M, (int)N, (int)K,
                                         (cudaStream_t)stream);
}

cudaError_t w4host::gemv_device_status(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, w4::g_device_status, sizeof *flag);
    if (e == cudaSuccess && *flag != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(w4::g_device_status, &zero, sizeof zero);
    }
    return e;
}
