// w4_gemv.cu -- decode-shaped W4A16 GEMM (few activation rows) on the
// warp-level MMA path.
//
// What it computes (INT4 QAT blog, Fig. 4 and "zero-overhead unpacking";
// reportify.cn "量化感知训练" [32][35]):  Y[m, n] = sum_k X[m, k] * dq(W)[n, k],
// dq(W)[n, k] = bf16_rne(q[n, k] * S[n, k/32]), FP32 accumulation, one BF16
// rounding of the result -- the product of w4_gemm.cu, for activation heights
// where the stream of packed weights from HBM, not the math, sets the time.
//
// Design (B200-first):
//  * one CTA per SM owns a contiguous range of output rows (cut at 4-row
//    granularity, so every SM streams the same number of bytes) and all of K
//    for them: no partial sum leaves the SM and no second kernel is needed;
//  * stages of (rows x K range) packed words and scales stream into a ring of
//    shared-memory slots, one 3-D TMA box each (64-byte swizzle on the words,
//    which makes the per-word row reads below free of bank conflicts); the
//    last warp done with a slot refills it, so no warp is spent on the loads
//    and no warp waits on another to start a copy;
//  * 16 compute warps split K: warp w owns one 128-wide K chunk per pass and
//    keeps that chunk of the activations in registers, already in MMA
//    B-fragment order; per stage it reads its chunk of a 16-row tile from
//    shared memory, unpacks the codes in registers (LOP3 + two packed BF16 ops
//    per pair of codes, the same exact dequant as the tensor-memory path)
//    straight into MMA A fragments and issues mma.sync m16n8k16 (BF16 in, FP32
//    accumulate), swap-AB: weight rows are the MMA's M, tokens its N.  Lane
//    (g, t) of a warp owns packed words t, t + 4, t + 8, t + 12 of a row's
//    chunk, so the four lanes of a token read 64 contiguous activation bytes
//    per load;
//  * the compute warps park their partial sums of a stage in one of four
//    shared-memory buffers and go on; a 17th warp adds them up in a fixed
//    order (deterministic), rounds and stores Y, so the compute warps never
//    wait for one another; a K longer than one pass of the warps keeps per-row
//    sums in shared memory between passes;
//  * 1..8 activation rows (one MMA N tile); the template also builds 16
//    (two tiles), which B200 measurements put behind the tensor-memory kernel.
// Inside an MMA the K order follows the packed word (codes j and j + 4 share a
// register) and the activation fragments are built in the same order; the K
// sum does not depend on the order of its terms.
// Every mbarrier wait is bounded (w4_common.cuh); a timed-out CTA records the
// device status, lets its issued copies land and exits.
#include <algorithm>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kGvWarps = 16;                          // compute warps
constexpr int kGvThreads = 32 * (kGvWarps + 1);       // + the reduction warp
constexpr int kGvKW = 128;                            // K of one warp chunk (4 groups)
constexpr int kGvWPT = 4;                             // packed words per lane, row and chunk

template <int NT, int RT, bool ZP = false>
struct GvCfg {
    static constexpr int MT = 8 * NT;                 // token columns (MMA N = 8 per tile)
    static constexpr int TPW = 1;                     // 16-row tiles per warp and stage
    static constexpr int KCW = kGvWarps / RT;         // K chunks per pass
    static constexpr int ROWS = 16 * TPW * RT;        // weight rows per stage
    static constexpr int WBYTES = KCW * ROWS * 64;    // packed words of a stage
    static constexpr int SKB = KCW / 2;               // 256-wide K blocks of scales per stage
    static constexpr int SBYTES = SKB * ROWS * 16;    // scales of a stage
    // zero points (ZP): 16-byte lines of 16 groups (512 of K) per row
    static constexpr int ZKB = KCW / 4;               // 512-wide K blocks per stage
    static constexpr int ZBYTES = ZP ? ZKB * ROWS * 16 : 0;
    static constexpr int NSTAGE = WBYTES >= 32768 ? 4 : 6;
    static_assert(NT == 1 || NT == 2, "at most 16 token columns per launch");
    static constexpr int PROWS = 16 * TPW;            // rows of one warp's partial tile
    static constexpr int TS = PROWS + 4;              // floats per token row (bank spread)
    static constexpr int RED_FLOATS = kGvWarps * MT * TS;      // one partial buffer
    static constexpr int NRED = 4;
    static constexpr int FIXED_BYTES =
        1024 + NSTAGE * (WBYTES + SBYTES + ZBYTES) + NRED * RED_FLOATS * 4;
    static_assert(WBYTES % 1024 == 0 && SBYTES % 128 == 0, "slot alignment");
    static_assert((ROWS * 64) % 512 == 0, "64-byte swizzle atoms");
    static_assert(KCW % 2 == 0, "chunk pairs share a scale block");
    static_assert(!ZP || KCW % 4 == 0, "chunk quads share a zero-point line");
};

struct GemvParams {
    const uint16_t *X;    // [M, K] BF16
    uint16_t *Y;          // [M, N] BF16
    int M, N, K;
    int n_quads, ctas;    // 4-row groups of N, CTAs they are cut over
    int kc, passes;       // K chunks, passes of the warps over them
    int acc_rows;         // row capacity of the cross-pass sums (0 when passes == 1)
};

__device__ __forceinline__ uint32_t gv_lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint2 gv_lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 gv_ldg128(const uint16_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t gv_atom_add_acq_rel(uint32_t addr, uint32_t v) {
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
__device__ __forceinline__ bool gv_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    const bool ok = mbar_wait(bar, parity, abort_flag);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Wait on the way out (ignores the abort flag): lets issued copies land.
__device__ __forceinline__ void gv_drain(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1; !mbar_try_wait(bar, parity); ++n) {
        if (n % kPollsPerCheck == 0 && globaltimer_ns() - t0 > kWaitLimitNs / 4) {
            record_timeout();
            return;
        }
    }
}

// Byte offset of packed word 4 j + t of line r in a chunk block of 64-byte
// lines with the TMA 64-byte swizzle (16-byte unit index ^= (r >> 1) & 3).
__device__ __forceinline__ uint32_t gv_word_off(int r, int j, int t) {
    return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4) + (t << 2));
}

// One stage of one warp: its K chunk of TPW 16-row tiles times the activation
// fragments xf, accumulated into acc.
//   lane (g, t), row r, word j: packed word 4 j + t of the chunk, i.e. K =
//   chunk * 128 + 32 j + 8 t + (0..7), scale group j of the chunk;
//   MMA step 2 j uses code pairs (0,4), (1,5); step 2 j + 1 uses (2,6), (3,7),
// matching the B fragments built by permute_chunk8 from the same 8 activations.
template <int NT, int TPW, bool ZP = false>
__device__ __forceinline__ void gv_stage_math(uint32_t wblk, uint32_t sblk, uint32_t zblk, int tile0, int g,
                                              int t, const uint4 (&xf)[NT][kGvWPT],
                                              float (&acc)[TPW][NT][4]) {
    // words j even / odd accumulate into two chains (half the dependent MMA
    // latency per stage), added at the end
    float acc2[TPW][NT][4];
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc2[u][nt][0] = acc2[u][nt][1] = acc2[u][nt][2] = acc2[u][nt][3] = 0.f;
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
        const int rg = (tile0 + u) * 16 + g, rh = rg + 8;
        uint32_t wg[kGvWPT], wh[kGvWPT];
#pragma unroll
        for (int j = 0; j < kGvWPT; ++j) {
            wg[j] = gv_lds32(wblk + gv_word_off(rg, j, t));
            wh[j] = gv_lds32(wblk + gv_word_off(rh, j, t));
        }
        // groups 0..3 of the chunk for rows rg and rh
        const uint2 sg = gv_lds64(sblk + (uint32_t)rg * 16);
        const uint2 sh = gv_lds64(sblk + (uint32_t)rh * 16);
        const uint32_t sgv[4] = {__byte_perm(sg.x, 0, 0x1010), __byte_perm(sg.x, 0, 0x3232),
                                 __byte_perm(sg.y, 0, 0x1010), __byte_perm(sg.y, 0, 0x3232)};
        const uint32_t shv[4] = {__byte_perm(sh.x, 0, 0x1010), __byte_perm(sh.x, 0, 0x3232),
                                 __byte_perm(sh.y, 0, 0x1010), __byte_perm(sh.y, 0, 0x3232)};
        // zero points of groups 0..3 (one byte each) for rows rg and rh
        const uint32_t zg = ZP ? gv_lds32(zblk + (uint32_t)rg * 16) : 0u;
        const uint32_t zh = ZP ? gv_lds32(zblk + (uint32_t)rh * 16) : 0u;
#pragma unroll
        for (int j = 0; j < kGvWPT; ++j) {
            uint32_t pg[4], ph[4];
            if (ZP) {
                dequant_word_k8perm_zp(wg[j], sgv[j], zp_bias2(zg >> (8 * j)), pg);
                dequant_word_k8perm_zp(wh[j], shv[j], zp_bias2(zh >> (8 * j)), ph);
            } else {
                dequant_word_k8perm(wg[j], sgv[j], pg);
                dequant_word_k8perm(wh[j], shv[j], ph);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float (&d)[4] = (j & 1) ? acc2[u][nt] : acc[u][nt];
                mma_bf16_m16n8k16(d, pg[0], ph[0], pg[1], ph[1], xf[nt][j].x, xf[nt][j].y);
                mma_bf16_m16n8k16(d, pg[2], ph[2], pg[3], ph[3], xf[nt][j].z, xf[nt][j].w);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[u][nt][e] += acc2[u][nt][e];
}

template <int NT, int RT, bool ZP>
__global__ void __launch_bounds__(kGvThreads, 1)
    w4a16_gemv_kernel(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap ts,
                      const __grid_constant__ CUtensorMap tz, const GemvParams p) {
    using C = GvCfg<NT, RT, ZP>;
    extern __shared__ __align__(1024) uint8_t gv_smem[];
    __shared__ __align__(8) uint64_t full_bar[C::NSTAGE];       // stage landed (TMA bytes)
    __shared__ __align__(8) uint64_t red_full[C::NRED];         // partials of a stage written
    __shared__ __align__(8) uint64_t red_empty[C::NRED];        // partials of a stage reduced
    __shared__ uint32_t slot_done[C::NSTAGE];                   // warps done with a slot
    __shared__ int slot_last[C::NSTAGE];                        // last stage issued to a slot
    __shared__ int abort_flag;

    const uint32_t raw = smem_u32(gv_smem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sm_w = base;
    const uint32_t sm_s = sm_w + C::NSTAGE * C::WBYTES;
    const uint32_t sm_z = sm_s + C::NSTAGE * C::SBYTES;     // ZP only
    const uint32_t sm_red = sm_z + C::NSTAGE * C::ZBYTES;
    float *red = reinterpret_cast<float *>(gv_smem + (sm_red - raw));
    float *rowsum = red + C::NRED * C::RED_FLOATS;    // [MT][acc_rows], passes > 1 only

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = (int)((int64_t)blockIdx.x * p.n_quads / p.ctas);
    const int q1 = (int)((int64_t)(blockIdx.x + 1) * p.n_quads / p.ctas);
    const int row0 = 4 * q0;
    const int row_end = min(p.N, 4 * q1);
    const int nrb = (row_end - row0 + C::ROWS - 1) / C::ROWS;
    const int nstages = nrb * p.passes;

    // stage s (pass-major, then row blocks) into slot s % NSTAGE
    auto issue = [&](int s) {
        const int slot = s % C::NSTAGE, pass = s / nrb, rb = s % nrb;
        const uint32_t fb = smem_u32(&full_bar[slot]);
        slot_last[slot] = s;
        mbar_arrive_expect_tx(fb, (uint32_t)(C::WBYTES + C::SBYTES + C::ZBYTES));
        tma_load_3d(sm_w + slot * C::WBYTES, &tw, fb, 0, row0 + rb * C::ROWS, pass * C::KCW);
        tma_load_3d(sm_s + slot * C::SBYTES, &ts, fb, 0, row0 + rb * C::ROWS, pass * C::SKB);
        if (ZP)
            tma_load_3d(sm_z + slot * C::ZBYTES, &tz, fb, 0, row0 + rb * C::ROWS, pass * C::ZKB);
    };
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tw);
        tma_prefetch_desc(&ts);
        if (ZP) tma_prefetch_desc(&tz);
        for (int i = 0; i < C::NSTAGE; ++i) {
            mbar_init(smem_u32(&full_bar[i]), 1u);
            slot_done[i] = 0u;
            slot_last[i] = -1;
        }
        for (int i = 0; i < C::NRED; ++i) {
            mbar_init(smem_u32(&red_full[i]), (uint32_t)kGvWarps);
            mbar_init(smem_u32(&red_empty[i]), 1u);
        }
        abort_flag = 0;
        fence_mbar_init();
        for (int i = 0; i < min(nstages, C::NSTAGE); ++i) issue(i);
    }
    __syncthreads();

    if (warp == kGvWarps) {
        // ---- reduction warp: stage s's partials, summed over the K chunks in a
        // fixed order, 4 consecutive rows x 1 token per item
        constexpr int ITEMS = RT * C::MT * 4;
        for (int s = 0; s < nstages; ++s) {
            const int b = s % C::NRED, pass = s / nrb, rb = s % nrb;
            const int n_active = min(C::KCW, p.kc - pass * C::KCW);
            if (!gv_wait(smem_u32(&red_full[b]), (uint32_t)((s / C::NRED) & 1), &abort_flag)) break;
            const float *rbuf = red + b * C::RED_FLOATS;
            for (int it = lane; it < ITEMS; it += 32) {
                const int i4 = 4 * (it & 3), t = (it >> 2) % C::MT, r_g = it / (4 * C::MT);
                const float *src = rbuf + r_g * C::KCW * (C::MT * C::TS) + t * C::TS + i4;
                // all loads first (unrolled, predicated), then the adds in chunk order
                float4 v[C::KCW];
#pragma unroll
                for (int c = 0; c < C::KCW; ++c)
                    v[c] = c < n_active ? *reinterpret_cast<const float4 *>(src + c * (C::MT * C::TS))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                float4 sum = v[0];
#pragma unroll
                for (int c = 1; c < C::KCW; ++c) {
                    sum.x += v[c].x;
                    sum.y += v[c].y;
                    sum.z += v[c].z;
                    sum.w += v[c].w;
                }
                const int rloc = rb * C::ROWS + r_g * 16 + i4;
                float sv[4] = {sum.x, sum.y, sum.z, sum.w};
                if (p.passes > 1) {
                    float *a = rowsum + t * p.acc_rows + rloc;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (pass > 0) sv[e] = a[e] + sv[e];
                        a[e] = sv[e];
                    }
                    if (pass + 1 < p.passes) continue;
                }
                if (t < p.M) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int n = row0 + rloc + e;
                        if (n < row_end) {
                            const __nv_bfloat16 v = __float2bfloat16_rn(sv[e]);
                            p.Y[(size_t)t * p.N + n] = *reinterpret_cast<const uint16_t *>(&v);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&red_empty[b]));
        }
    } else {
        // ---- compute warps
        const int g = lane >> 2, tig = lane & 3;
        const int rt = warp / C::KCW, cw = warp % C::KCW;
        uint4 xf[NT][kGvWPT];
        for (int pass = 0; pass < p.passes; ++pass) {
            const int chunk = pass * C::KCW + cw;
            const bool active = cw < min(C::KCW, p.kc - pass * C::KCW);
            // this chunk of the activations, in B-fragment order (rows >= M are
            // zero): lane (g, t) holds token g's K = chunk * 128 + 32 j + 8 t + (0..7)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = 8 * nt + g;
#pragma unroll
                for (int j = 0; j < kGvWPT; ++j) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (active && tok < p.M)
                        v = gv_ldg128(p.X + (size_t)tok * p.K + (size_t)chunk * kGvKW + 32 * j +
                                      8 * tig);
                    xf[nt][j] = permute_chunk8(v);
                }
            }
            for (int rb = 0; rb < nrb; ++rb) {
                const int s = pass * nrb + rb;
                const int slot = s % C::NSTAGE;
                const bool ok = gv_wait(smem_u32(&full_bar[slot]), (uint32_t)((s / C::NSTAGE) & 1),
                                        &abort_flag);
                float acc[C::TPW][NT][4];
#pragma unroll
                for (int u = 0; u < C::TPW; ++u)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        acc[u][nt][0] = acc[u][nt][1] = acc[u][nt][2] = acc[u][nt][3] = 0.f;
                if (ok && active) {
                    const uint32_t wblk = sm_w + slot * C::WBYTES + cw * (C::ROWS * 64);
                    const uint32_t sblk =
                        sm_s + slot * C::SBYTES + (cw >> 1) * (C::ROWS * 16) + (cw & 1) * 8;
                    const uint32_t zblk =
                        sm_z + slot * C::ZBYTES + (cw >> 2) * (C::ROWS * 16) + (cw & 3) * 4;
                    gv_stage_math<NT, C::TPW, ZP>(wblk, sblk, zblk, rt * C::TPW, g, tig, xf, acc);
                }
                // The math has consumed this warp's reads of the slot; the last
                // warp done with it (the counter only grows: 16 arrivals per use)
                // refills it with stage s + NSTAGE.
                __syncwarp();
                if (lane == 0) {
                    const uint32_t before = gv_atom_add_acq_rel(smem_u32(&slot_done[slot]), 1u);
                    if (before == (uint32_t)(kGvWarps * (s / C::NSTAGE + 1) - 1) &&
                        s + C::NSTAGE < nstages && !abort_flag)
                        issue(s + C::NSTAGE);
                }
                // partial sums of this warp: [token][row of its tile], TS floats per token
                const int b = s % C::NRED;
                bool ok_red = true;
                if (s >= C::NRED)
                    ok_red = gv_wait(smem_u32(&red_empty[b]), (uint32_t)((s / C::NRED - 1) & 1),
                                     &abort_flag);
                float *buf = red + b * C::RED_FLOATS + warp * (C::MT * C::TS);
                if (active && ok_red) {
#pragma unroll
                    for (int u = 0; u < C::TPW; ++u)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int t = 8 * nt + 2 * tig, i = 16 * u + g;
                            buf[t * C::TS + i] = acc[u][nt][0];
                            buf[(t + 1) * C::TS + i] = acc[u][nt][1];
                            buf[t * C::TS + i + 8] = acc[u][nt][2];
                            buf[(t + 1) * C::TS + i + 8] = acc[u][nt][3];
                        }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&red_full[b]));
            }
        }
    }
    // after a timeout: every issued copy lands before the shared memory goes away
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag)
        for (int i = 0; i < C::NSTAGE; ++i)
            if (slot_last[i] >= 0)
                gv_drain(smem_u32(&full_bar[i]), (uint32_t)((slot_last[i] / C::NSTAGE) & 1));
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int NT, int RT, bool ZP = false>
w4_status gv_launch(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z,
                    w4_bf16 *Y, int M, int N, int K, cudaStream_t stream) {
    using C = GvCfg<NT, RT, ZP>;
    const int sms = w4host::num_sms();
    GemvParams p = {};
    p.X = reinterpret_cast<const uint16_t *>(X);
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    p.n_quads = (N + 3) / 4;
    // at least one 16-row tile per CTA
    p.ctas = std::max(1, std::min(sms, (N + 15) / 16));
    p.kc = K / kGvKW;
    p.passes = (p.kc + C::KCW - 1) / C::KCW;
    const int max_rows = 4 * ((p.n_quads + p.ctas - 1) / p.ctas);
    p.acc_rows = p.passes > 1 ? (max_rows + C::ROWS - 1) / C::ROWS * C::ROWS : 0;
    const size_t smem = (size_t)C::FIXED_BYTES + (size_t)p.acc_rows * C::MT * 4;
    if (smem > 225 * 1024) return W4_ERR_UNSUPPORTED;

    CUtensorMap tw, ts, tz;
    {
        // packed words as [K / 128 chunks][N rows][16 words]; the chunk stride
        // (one 64-byte line) is smaller than the row stride
        cuuint64_t dims[3] = {16u, (cuuint64_t)N, (cuuint64_t)(K / kGvKW)};
        cuuint64_t strides[2] = {(cuuint64_t)K / 2, 64u};
        cuuint32_t box[3] = {16u, (cuuint32_t)C::ROWS, (cuuint32_t)C::KCW};
        if (w4host::encode_tiled(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, const_cast<int32_t *>(Wq),
                                 dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    {
        // scales as [K / 256 blocks][N rows][8 groups]
        cuuint64_t dims[3] = {8u, (cuuint64_t)N, (cuuint64_t)(K / 256)};
        cuuint64_t strides[2] = {(cuuint64_t)K / 16, 16u};
        cuuint32_t box[3] = {8u, (cuuint32_t)C::ROWS, (cuuint32_t)C::SKB};
        if (w4host::encode_tiled(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<w4_bf16 *>(S),
                                 dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    if (ZP) {
        // zero points as [K / 512 blocks][N rows][16 groups], one byte each
        cuuint64_t dims[3] = {16u, (cuuint64_t)N, (cuuint64_t)(K / 512)};
        cuuint64_t strides[2] = {(cuuint64_t)K / 32, 16u};
        cuuint32_t box[3] = {16u, (cuuint32_t)C::ROWS, (cuuint32_t)C::ZKB};
        if (w4host::encode_tiled(&tz, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(Z),
                                 dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    } else {
        tz = ts;                                     // not read
    }
    auto kern = w4a16_gemv_kernel<NT, RT, ZP>;
    static size_t configured = 0;
    if (smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return w4host::launch_status();
        configured = smem;
    }
    kern<<<p.ctas, kGvThreads, smem, stream>>>(tw, ts, tz, p);
    return w4host::launch_status();
}

}  // namespace
}  // namespace w4

// Shapes the warp-level MMA path takes: 1..8 activation rows (measured on
// B200: from 16 rows on, the tensor-memory kernel is faster), K a multiple of
// 256 (whole 256-wide scale blocks per TMA box).
bool w4host::gemv_supported(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && M <= 8 && N >= 1 && N <= (1 << 30) && K >= 256 && (K % 256) == 0 &&
           K <= (1 << 24);
}

w4_status w4host::gemv_launch(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, w4_bf16 *Y,
                              int64_t M, int64_t N, int64_t K, void *stream) {
    using namespace w4;
    if (!gemv_supported(M, N, K)) return W4_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    const int m = (int)M, n = (int)N, k = (int)K;
    // short K (at most 8 chunks of 128): two row tiles of warps per stage
    return k / kGvKW <= 8 ? gv_launch<1, 2>(X, Wq, S, nullptr, Y, m, n, k, st)
                          : gv_launch<1, 1>(X, Wq, S, nullptr, Y, m, n, k, st);
}

w4_status w4host::gemv_launch_zp(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                                 const uint8_t *Z, w4_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                 void *stream) {
    using namespace w4;
    if (!gemv_supported(M, N, K) || (K % 512) != 0 || !aligned16(Z)) return W4_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    const int m = (int)M, n = (int)N, k = (int)K;
    return k / kGvKW <= 8 ? gv_launch<1, 2, true>(X, Wq, S, Z, Y, m, n, k, st)
                          : gv_launch<1, 1, true>(X, Wq, S, Z, Y, m, n, k, st);
}

cudaError_t w4host::gemv_device_status(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, w4::g_device_status, sizeof *flag);
    if (e == cudaSuccess && *flag != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(w4::g_device_status, &zero, sizeof zero);
    }
    return e;
}
