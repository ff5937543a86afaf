// w4_gemm.cu -- W4A16 GEMM (dense) and grouped MoE W4A16 GEMM on 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// What it computes (INT4 QAT blog, Fig. 4 and "zero-overhead unpacking";
// reportify.cn "量化感知训练" [32][35]):  Y[m, n] = sum_k X[m, k] * dq(W)[n, k],
// dq(W)[n, k] = bf16_rne(q[n, k] * S[n, k/32]), FP32 accumulation, one BF16
// rounding of the result.  The MoE variant runs the same product per aligned
// block of slots with the block's expert weights and gathered activation rows.
// Two more weight prologues share the tile: BF16 weights through the exact
// group QDQ of the quantizers (QAT forward, Y = X . fake_quant(W)^T), and
// unsigned codes with a zero point per group, dq = bf16_rne((q - z) * s)
// (quantization tutorial §2.1 / §2.3), and micro-scaled FP4 codes (MR-GPTQ /
// QuTLASS FP4 summary: MXFP4, E2M1 with a power-of-two scale per 32; NVFP4,
// E2M1 with an E4M3 scale per 16 under an FP32 tensor scale), which keep the
// activations in BF16.
//
// Design (B200-first; the pages' Marlin kernel targets H-series mma.sync and
// is prior art only):
//  * swap-AB: the MMA's A operand (M = 128 rows) is the dequantized weight
//    tile, the B operand (N = MT columns) is the activation tile, so decode
//    shapes with 1..64 tokens still use a full-height MMA;
//  * the weights never exist as BF16 in memory or shared memory: packed words
//    arrive by TMA (128-byte swizzle, bank-conflict-free row reads), dequant
//    warps unpack them in registers (LOP3 + 2 packed BF16 ops per pair of
//    codes) and store the BF16 A tile straight into tensor memory with
//    tcgen05.st; tcgen05.mma then reads A from TMEM and B from shared memory,
//    which keeps the shared-memory traffic of a decode step at the packed
//    bytes plus the activations;
//  * with 256-wide k-blocks a register pair holds codes (j, j + 4) of a packed
//    word, which saves the PRMT that natural order needs; two activation-
//    reorder warps permute the activation chunks in shared memory to match,
//    overlapped with the unpacking of the same stage;
//  * activations arrive by TMA in the canonical K-major 128-byte-swizzled
//    layout (dense), or by cp.async row gathers into the same layout (MoE);
//  * warp specialization: warp 0 = loads + TMEM allocation, then groups of
//    four dequant warps that take turns over the k-blocks, then four epilogue
//    warps and the MMA issuers (several where one thread cannot keep up: it
//    issues a tcgen05.mma only every ~100 cycles; each issuer owns its own
//    accumulator and every NSPLIT-th K step, or, for the 256-token tiles, its
//    own token range of one accumulator at every K step), with mbarrier rings
//    between the roles;
//  * persistent CTAs (one per SM) walk a static list of work items.  A decode
//    GEMM given a workspace splits the (row tile, k-block) units evenly over
//    the SMs (stream-K); the last CTA to finish a row tile adds the parked
//    FP32 partial sums in ascending K order, so the result is deterministic.
//    Without a workspace the N rows are split evenly (rows per tile =
//    ceil(N / SMs)) and no reduction is needed.
// Every mbarrier wait is bounded (w4_common.cuh); a timed-out CTA records the
// device status, drains its own in-flight copies and MMAs, frees its TMEM and
// exits.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "w4_common.cuh"
#include "w4_qdq.cuh"

namespace w4 {
namespace {

// Warp roles: warp 0 = loads (and TMEM allocation), then 4 * NDQ dequant warps
// (NDQ groups of four that take turns over the k-blocks), then (256-wide
// k-blocks only) kPermWarps warps that reorder the activation chunks, then
// 4 epilogue warps (each drains the accumulators of its TMEM lane quarter),
// then NSPLIT MMA issuer warps: lane 0 of issuer i issues every NSPLIT-th
// 16-wide K step into accumulator i.  A thread issues a tcgen05.mma only about
// every 100 cycles (issue latency, not the tensor core), and each k-block adds
// a barrier poll and two commits, so small-N tiles need several issuers to
// keep up with HBM.
__host__ __device__ constexpr int perm_warps(int kb) { return kb == 256 ? 2 : 0; }
__host__ __device__ constexpr int gemm_threads(int ndq, int kb, int nsplit, bool wgl) {
    return wgl ? 128 * (ndq + 4) : 32 * (1 + 4 * ndq + perm_warps(kb) + 4 + nsplit);
}
// Warpgroup layout (WGL, for the decode tiles that need eight issuers): aligned
// warpgroups of four warps, each resizing its register file with setmaxnreg:
//   WG 0 .. NDQ-1: dequant groups;  WG NDQ: epilogue;  WG NDQ+1, NDQ+2: up to
//   eight MMA issuers;  WG NDQ+3: loads (warp 0, also the TMEM allocation) and
//   the activation reorder (the next kPermWarps warps).
// Each SM sub-partition holds one warp of every warpgroup, so its register
// file is shared by ndq + 4 warps at launch; the dequant warpgroups take what
// the others give back.
__host__ __device__ constexpr int launch_regs_wgl(int ndq) {
    return 16384 / (32 * (ndq + 4)) / 8 * 8;
}
constexpr int kRegsEpi = 88, kRegsIssue = 40, kRegsLoad = 64;
__host__ __device__ constexpr int dequant_regs_wgl(int ndq) {
    return (launch_regs_wgl(ndq) * (ndq + 4) - kRegsEpi - 2 * kRegsIssue - kRegsLoad) / ndq / 8 *
           8;
}
// registers the split takes per sub-partition lane slot (checked on the host
// against what the launch allocates: setmaxnreg.inc would wait forever otherwise)
__host__ __device__ constexpr int split_regs_wgl(int ndq) {
    return ndq * dequant_regs_wgl(ndq) + kRegsEpi + 2 * kRegsIssue + kRegsLoad;
}
constexpr int kTmemCols = 512;

struct GemmParams {
    const uint16_t *S;           // scales (direct loads when KB < 256)
    const uint8_t *Z;            // zero points of asymmetric groups (ZP), one byte per group;
                                 // FP4: the group scale bytes (E8M0 or E4M3)
    float fp4_g;                 // NVFP4: the FP32 tensor scale
    uint16_t *Y;                 // dense: Y [M, N]; MoE: C [num_slots, N]
    const uint16_t *A;           // MoE: activation rows [a_rows, K]
    const int32_t *sorted_ids;   // MoE
    const int32_t *expert_ids;   // MoE
    const int32_t *num_post_pad; // MoE
    int64_t M, N, K;
    int64_t num_slots;           // MoE
    int64_t a_rows;              // MoE
    int a_row_div;               // MoE
    int cap_blocks;              // MoE: length of expert_ids (bounds num_post_pad / block)
    int moe_sub;                 // MoE: MT-slot sub-blocks per aligned block (block / MT)
    int moe_mt;                  // MoE: MT (slots per work item)
    // MoE down projection with the weighted top-k combine fused: out [T, N] =
    // sum_k w[t, k] * C[t * topk + k, :], done by the last work item to finish
    // a token's row tile (arrival counters per token, row tile, lane quarter)
    const float *comb_w;         // [T, topk] FP32 routing weights
    uint16_t *comb_out;          // [T, N] BF16; nullptr: no combine
    unsigned int *comb_cnt;      // [T][n_row_tiles][4], zero between calls
    int topk;
    int silu_inter;              // MoE gate_up with SiLU*up fused: the intermediate
                                 // size F (weights [E, 2F, K]; Y = H [num_slots, F]);
                                 // 0 = plain grouped GEMM
    int rows_per_tile;           // R <= 128
    int n_row_tiles;
    int n_tok_tiles;             // dense
    int num_kb;
    // stream-K split of the (row tile, k-block) units of a one-token-tile GEMM
    int split;                   // 0: whole-K work items; 1: split units
    int64_t units;               // n_row_tiles * num_kb
    int ctas;                    // grid size the split was planned for
    int max_contrib;             // most CTAs sharing one row tile
    float *ws_part;              // [n_row_tiles][max_contrib][128][MT] partial sums
    unsigned int *ws_cnt;        // [n_row_tiles][4] arrival counters (zero between calls)
};

// Work items: (row tile rt, token tile tt, k-blocks [kb0, kb1)).  Dense and MoE
// kernels walk whole-K items blockIdx.x, blockIdx.x + gridDim.x, ...; a split
// kernel walks the CTA's contiguous range of (row tile, k-block) units, cut at
// row-tile boundaries.
// 32-bit unsigned arithmetic throughout: the host enables the split only when
// units * (ctas + 1) < 2^32, and the item count of the other modes is an int.
struct ItemIter {
    uint32_t cur, end, step;
};

__device__ __forceinline__ ItemIter make_iter(const GemmParams &p, int num_items) {
    ItemIter I;
    if (p.split) {
        const uint32_t units = (uint32_t)p.units, ctas = (uint32_t)p.ctas;
        I.cur = blockIdx.x * units / ctas;
        I.end = (blockIdx.x + 1) * units / ctas;
        I.step = 0;
    } else {
        I.cur = blockIdx.x;
        I.end = (uint32_t)num_items;
        I.step = gridDim.x;
    }
    return I;
}

__device__ __forceinline__ bool next_item(ItemIter &I, const GemmParams &p, int &rt, int &tt,
                                          int &kb0, int &kb1) {
    if (I.cur >= I.end) return false;
    if (p.split) {
        // The CTA's units [a, b) touch at most two row tiles (fewer units than
        // k-blocks per tile).  The piece in the later tile (its first k-blocks)
        // goes first: its partial sums are parked early, while the CTA works on
        // the piece in the earlier tile (that tile's last k-blocks), which the
        // previous CTA started first, so this CTA usually arrives last there and
        // does the tile's fixup at its end with the other partials already
        // parked.  I.step: 0 = later piece next, 1 = earlier piece next.
        const uint32_t nkb = (uint32_t)p.num_kb;
        const uint32_t a = I.cur, b = I.end;
        const uint32_t t1 = (b - 1) / nkb;
        const uint32_t split_at = max(a, t1 * nkb);
        if (I.step == 0) {
            rt = (int)t1;
            kb0 = (int)(split_at - t1 * nkb);
            kb1 = (int)(b - t1 * nkb);
            I.step = 1;
            if (split_at == a) I.cur = I.end;       // a single piece
        } else {
            const uint32_t t0 = a / nkb;
            rt = (int)t0;
            kb0 = (int)(a - t0 * nkb);
            kb1 = (int)(split_at - t0 * nkb);
            I.cur = I.end;
        }
        tt = 0;
    } else {
        const uint32_t nrt = (uint32_t)p.n_row_tiles;
        for (;;) {
            const uint32_t q = I.cur / nrt;
            rt = (int)(I.cur - q * nrt);
            tt = (int)q;
            I.cur += I.step;
            // MoE: a sub-block whose first slot is padding is padding throughout
            // (an expert's run holds its real slots first); every role skips it
            if (p.sorted_ids == nullptr || p.moe_sub == 1) break;
            const int32_t first = __ldg(p.sorted_ids + (int64_t)tt * p.moe_mt);
            if (first >= 0 && first < p.num_slots) break;
            if (I.cur >= I.end) return false;
        }
        kb0 = 0;
        kb1 = p.num_kb;
    }
    return true;
}

__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int *p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// CTA that owns split unit x (CTA c owns [c*U/P, (c+1)*U/P)).
__device__ __forceinline__ int unit_owner(uint32_t x, const GemmParams &p) {
    return (int)(((x + 1) * (uint32_t)p.ctas - 1) / (uint32_t)p.units);
}

// Shared-memory layout, all offsets from a 1024-aligned base.
template <int KB, int MT, int NSTAGE, int NACC, int NASTAGE, int NSPLIT, bool BF16W = false,
          bool SMEM_A = false, bool A_IN_TMEM = true>
struct Layout {
    // weight tile of up to 128 rows: packed INT4 words, or BF16 weights (QAT)
    static constexpr int kWBytes = BF16W ? 128 * KB * 2 : 128 * KB / 2;
    static constexpr int kSBytes = (KB == 256) ? 128 * 16 : 0;
    static constexpr int kXSub = MT * 128;                  // one 64-wide K slice
    static constexpr int kXBytes = (KB / 64) * kXSub;
    static constexpr int kStage = kWBytes + kSBytes + kXBytes;
    // A operand in shared memory (QAT input gradient): NASTAGE BF16 tiles of
    // 128 rows x KB, K-major, 128-byte swizzle
    static constexpr int kAOff = NSTAGE * kStage;
    static constexpr int kASlot = 128 * KB * 2;
    static constexpr int kBarOff = kAOff + (SMEM_A ? NASTAGE * kASlot : 0);
    static constexpr int kNumBars = 2 * NSTAGE + 2 * NASTAGE + 2 * NACC + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kAlloc = kBytes + 1024;            // slack for 1024-alignment
    static_assert(kWBytes % 1024 == 0 && kXSub % 1024 == 0, "1024-byte aligned tiles");
    static_assert(kStage % 1024 == 0, "stage size");
    static_assert(NACC * NSPLIT * MT + (A_IN_TMEM ? NASTAGE * (KB / 2) : 0) <= kTmemCols,
                  "TMEM budget");
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t swz(uint32_t off, uint32_t sw_bytes) {
    // TMA / UMMA swizzle: 16-byte chunk index XOR address bits [7, ...).
    return off ^ (((off >> 7) & (sw_bytes / 16 - 1)) << 4);
}

// Bounded wait executed by every lane of a warp; the verdict is warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t sleep_ns = kPollSleepNs) {
    bool ok = mbar_wait(bar, parity, abort_flag, sleep_ns);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Back-off per kind of waiter: the dequant warps and the MMA issuers are on the
// critical path (default back-off); the loads, the activation reorder and the
// accumulator hand-over run ahead of it; the epilogue waits a whole work item.
constexpr uint32_t kSleepAhead = 128;
constexpr uint32_t kSleepLong = 256;

// Drain wait used on the way out of an aborted CTA (does not look at the abort flag).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1; !mbar_try_wait(bar, parity); ++n) {
        if (n % kPollsPerCheck == 0 && globaltimer_ns() - t0 > kWaitLimitNs / 4) {
            record_timeout();
            return;
        }
    }
}

// NSPLIT: MMA issuers = accumulators per work item; 16-wide K step u goes to
// issuer / accumulator u % NSPLIT, and the epilogue adds the accumulators in
// a fixed order.  SPLITN: the NSPLIT issuers split the tile's tokens instead
// (issuer i: columns [i MT/NSPLIT, (i+1) MT/NSPLIT) of the one accumulator,
// every K step), so NSPLIT threads issue into one accumulator in parallel:
// one thread issues a tcgen05.mma only about every 100 cycles, and with a
// barrier poll and a commit per k-block a single issuer cannot keep up with
// the tensor core on N = 256 tiles.
template <int KB, int MT, int NSTAGE, int NACC, int NASTAGE, int NSPLIT, int NDQ, bool MOE,
          bool WGL, int QAT, bool ZP, bool SPLITN, int FP4>
__global__ void __launch_bounds__(gemm_threads(NDQ, KB, NSPLIT, WGL), 1)
    w4a16_tc_kernel(const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_s,
                    const __grid_constant__ CUtensorMap tm_x, const GemmParams p) {
    constexpr int kAccSets = SPLITN ? 1 : NSPLIT;   // accumulators per work item
    // QAT = 1: forward (fake quantization of W in the weight prologue, A in
    // TMEM); QAT = 2: input gradient dX = dY . fake_quant(W), A = fake_quant(W)^T
    // tile in shared memory; QAT = 3: forward with the QDQ written back in place
    // over the weight tile, which the MMA then reads as A from shared memory
    // (tensor memory holds only accumulators)
    constexpr bool kQdx = (QAT == 2);
    constexpr bool kQin = (QAT == 3);
    using L = Layout<KB, MT, NSTAGE, NACC, NASTAGE, kAccSets, (QAT != 0), kQdx, (QAT <= 1)>;
    static_assert(!QAT || (KB == 64 && !MOE && QAT <= 3),
                  "QAT: 64-wide k-blocks of dense BF16 weights");
    static_assert(!(kQdx || kQin) || NSTAGE == NASTAGE,
                  "A in shared memory: one release per k-block");
    static_assert(MT <= 256 || (SPLITN && MT / NSPLIT <= 256 && QAT >= 2),
                  "more than 256 tokens per item: token-split issuers, A in shared memory");
    static_assert(!SPLITN || (KB == 64 && !MOE && !WGL && MT % (16 * NSPLIT) == 0),
                  "token-split issuers: dense 64-wide k-blocks, N per issuer a multiple of 16");
    static_assert(!ZP || ((KB == 64 || KB == 256) && !MOE && !QAT),
                  "zero points: dense k-blocks");
    // FP4 = 1: MXFP4 (a scale byte per 32 codes), 2: NVFP4 (a scale byte per 16)
    static_assert(FP4 == 0 || ((KB == 64 || KB == 256) && !MOE && !QAT && !ZP && FP4 <= 2),
                  "FP4 codes: dense k-blocks");
    // 256-wide k-blocks with zero points or FP4 scales: the row's bytes of the
    // k-block (8 zero points / E8M0 scales, 16 E4M3 scales) are read directly
    // by the dequant warps; FP4 codes unpack in natural order, so the
    // activation chunks keep theirs (the reorder warps only join the barrier)
    constexpr bool kByteScales = (KB == 256) && (ZP || FP4 != 0);
    static_assert(!kByteScales || !WGL, "byte scales: flat warp layout");
    constexpr int kWords = KB / 8;             // packed words per row per k-block
    constexpr int kAStageCols = KB / 2;        // TMEM columns per A stage
    constexpr int kAccCols = kAccSets * MT;    // TMEM columns per work item accumulator
    constexpr int kNPer = SPLITN ? MT / NSPLIT : MT;   // MMA N of one issuer
    constexpr int kABase = NACC * kAccCols;    // first A column
    constexpr int kDqWarps = 4 * NDQ;
    constexpr int kPermWarps = perm_warps(KB);
    constexpr int kEpiWarp0 = 1 + kDqWarps + kPermWarps;
    constexpr int kWgLoad = NDQ + 3;                        // (warpgroup layout)
    constexpr int kAllocWarp = WGL ? 4 * kWgLoad : 0;      // loads + TMEM allocation
    static_assert(NSPLIT >= 1 && NSPLIT <= (WGL ? 8 : 4), "MMA issuers");
    static_assert(!WGL || (kPermWarps <= 3 && dequant_regs_wgl(NDQ) >= 96 &&
                           split_regs_wgl(NDQ) <= launch_regs_wgl(NDQ) * (NDQ + 4)),
                  "warpgroup register split");
    // 256-wide k-blocks (decode / MoE, few activation rows per tile): reorder the
    // activation chunks in shared memory instead of pairing the unpacked codes.
    constexpr bool kXPerm = (KB == 256);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, kNPer);

    extern __shared__ uint8_t smem_raw[];
    // MoE gate_up with SiLU*up: the up rows' sums of one 16-column chunk, handed
    // from the epilogue warps of lane quarters 2-3 to those of 0-1
    __shared__ __align__(16) float xchg[MOE ? 64 * 16 : 4];
    __shared__ __align__(8) uint64_t xchg_bar[2];     // [0] written, [1] read
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::kBarOff;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (NSTAGE + s); };
    auto afull_bar = [&](int a) { return bar0 + 8u * (2 * NSTAGE + a); };
    auto aempty_bar = [&](int a) { return bar0 + 8u * (2 * NSTAGE + NASTAGE + a); };
    // As many A slots as stages: k-block it uses stage and A slot it % NSTAGE,
    // both freed by the completion of its MMAs, so one commit (to the stage's
    // "empty" barrier) releases both, and the dequant warps wait on that one.
    constexpr bool kOneRelease = (NSTAGE == NASTAGE);
    auto aslot_free_bar = [&](uint32_t it) {
        return kOneRelease ? empty_bar((int)(it % NSTAGE)) : aempty_bar((int)(it % NASTAGE));
    };
    auto aslot_free_parity = [&](uint32_t it) { return ((it / NASTAGE) & 1u) ^ 1u; };
    auto accfull_bar = [&](int d) { return bar0 + 8u * (2 * NSTAGE + 2 * NASTAGE + d); };
    auto accempty_bar = [&](int d) {
        return bar0 + 8u * (2 * NSTAGE + 2 * NASTAGE + NACC + d);
    };
    const uint32_t mmadone_bar = bar0 + 8u * (2 * NSTAGE + 2 * NASTAGE + 2 * NACC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);

    auto w_stage = [&](int s) { return sbase + (uint32_t)(s * L::kStage); };
    auto s_stage = [&](int s) { return sbase + (uint32_t)(s * L::kStage + L::kWBytes); };
    auto x_stage = [&](int s) {
        return sbase + (uint32_t)(s * L::kStage + L::kWBytes + L::kSBytes);
    };
    auto a_smem = [&](int a) { return sbase + (uint32_t)(L::kAOff + a * L::kASlot); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(full_bar(s), MOE ? 33u : 1u);
            mbar_init(empty_bar(s), (uint32_t)NSPLIT);
        }
        for (int a = 0; a < NASTAGE; ++a) {
            // one dequant group, plus the activation-reorder warps
            mbar_init(afull_bar(a), 128u + (kXPerm ? 32u * kPermWarps : 0u));
            mbar_init(aempty_bar(a), (uint32_t)NSPLIT);
        }
        for (int d = 0; d < NACC; ++d) {
            mbar_init(accfull_bar(d), (uint32_t)NSPLIT);
            mbar_init(accempty_bar(d), 128u);
        }
        mbar_init(mmadone_bar, (uint32_t)NSPLIT);
        if (MOE) {
            mbar_init(smem_u32(&xchg_bar[0]), 2u);
            mbar_init(smem_u32(&xchg_bar[1]), 2u);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_w);
        if (KB == 256 && FP4 == 0) tma_prefetch_desc(&tm_s);
        if (!MOE) tma_prefetch_desc(&tm_x);
    }
    // Decode tiles: warm L2 with this CTA's first weight and scale tiles (its
    // work items follow from the parameters alone) while the kernel before it
    // drains; measured faster chained behind another GEMM, where the warp-level
    // decode kernel measured slower with the same prefetch.
    if (KB == 256 && !MOE && !QAT && threadIdx.x == 0) {
        ItemIter I = make_iter(p, p.n_row_tiles * p.n_tok_tiles);
        int rt, tt, kb0, kb1, left = 32;
        while (left > 0 && next_item(I, p, rt, tt, kb0, kb1))
            for (int kb = kb0; kb < kb1 && left > 0; ++kb, --left) {
                tma_prefetch_l2_2d(&tm_w, kb * kWords, rt * p.rows_per_tile);
                if (FP4 == 0) tma_prefetch_l2_2d(&tm_s, kb * 8, rt * p.rows_per_tile);
            }
    }
    // the kernel before this one on the stream may still be running: no global
    // memory (and no tensor memory, which a co-resident CTA of it may hold)
    // is touched before it completes
    griddep_wait();
    griddep_launch_dependents();
    if (warp == kAllocWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const int R = p.rows_per_tile;
    const int num_kb = p.num_kb;
    int num_items;
    if (MOE) {
        const int npp = *p.num_post_pad;
        const int nblocks = min(max(npp, 0) / MT, p.cap_blocks * p.moe_sub);
        num_items = nblocks * p.n_row_tiles;
    } else {
        num_items = p.n_row_tiles * p.n_tok_tiles;
    }

    // ---- role bodies (inlined at each call site below)
    auto role_loads = [&]() {
        // ------------------------------------------------------------ loads
        uint32_t it = 0;
        bool ok = true;
        ItemIter I = make_iter(p, num_items);
        int rt, tt, kb0, kb1;
        while (ok && next_item(I, p, rt, tt, kb0, kb1)) {
            const int row0 = rt * R;
            int expert = 0;
            // MoE: activation row of each of the block's MT slots (-1 for padding),
            // lane t % 32 of register t / 32, loaded once per work item
            int gather_row[(MT + 31) / 32];
            if (MOE) {
                expert = __ldg(p.expert_ids + tt / p.moe_sub);
#pragma unroll
                for (int r = 0; r < (MT + 31) / 32; ++r) {
                    const int t = r * 32 + lane;
                    int row = -1;
                    if (t < MT) {
                        const int slot = __ldg(p.sorted_ids + (int64_t)tt * MT + t);
                        if (slot >= 0 && slot < p.num_slots) {
                            row = slot / p.a_row_div;
                            if (row >= p.a_rows) row = -1;
                        }
                    }
                    gather_row[r] = row;
                }
            }
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % NSTAGE;
                if (!warp_wait(empty_bar(s), ((it / NSTAGE) & 1u) ^ 1u, abort_flag, kSleepAhead)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t wbytes = QAT ? (uint32_t)R * KB * 2u : (uint32_t)R * (KB / 2);
                    const uint32_t sbytes = (KB == 256 && FP4 == 0) ? (uint32_t)R * 16u : 0u;
                    const uint32_t xbytes = MOE ? 0u : (uint32_t)L::kXBytes;
                    mbar_arrive_expect_tx(full_bar(s), wbytes + sbytes + xbytes);
                    if (MOE && p.silu_inter > 0) {
                        // SiLU*up tile: rows 0-63 are gate rows rt*64 + i, rows
                        // 64-127 the matching up rows F + rt*64 + i (64-row boxes)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int grow = h * p.silu_inter + rt * 64;
                            tma_load_3d(w_stage(s) + (uint32_t)(64 * h) * (KB / 2), &tm_w,
                                        full_bar(s), kb * kWords, grow, expert);
                            if (KB == 256)
                                tma_load_3d(s_stage(s) + (uint32_t)(64 * h) * 16u, &tm_s,
                                            full_bar(s), kb * 8, grow, expert);
                        }
                    } else if (MOE) {
                        tma_load_3d(w_stage(s), &tm_w, full_bar(s), kb * kWords, row0, expert);
                        if (KB == 256)
                            tma_load_3d(s_stage(s), &tm_s, full_bar(s), kb * 8, row0, expert);
                    } else if (kQdx) {
                        // W [N, K] as two 64 x 64 boxes: K (output rows) row0 ..
                        // row0 + 127, N (the contraction) kb * 64 .. + 63
                        tma_load_2d(w_stage(s), &tm_w, full_bar(s), row0, kb * KB);
                        tma_load_2d(w_stage(s) + L::kWBytes / 2, &tm_w, full_bar(s), row0 + 64,
                                    kb * KB);
#pragma unroll
                        for (int h = 0; h < (MT + 255) / 256; ++h)
                            tma_load_2d(x_stage(s) + h * 256 * 128, &tm_x, full_bar(s), kb * KB,
                                        tt * MT + h * 256);
                    } else {
                        tma_load_2d(w_stage(s), &tm_w, full_bar(s), QAT ? kb * KB : kb * kWords,
                                    row0);
                        if (KB == 256 && FP4 == 0)
                            tma_load_2d(s_stage(s), &tm_s, full_bar(s), kb * 8, row0);
#pragma unroll
                        for (int u = 0; u < KB / 64; ++u)
#pragma unroll
                            for (int h = 0; h < (MT + 255) / 256; ++h)
                                tma_load_2d(x_stage(s) + u * L::kXSub + h * 256 * 128, &tm_x,
                                            full_bar(s), kb * KB + u * 64, tt * MT + h * 256);
                    }
                }
                if (MOE) {
                    // Gather the block's activation rows: lane = 16-byte chunk along K;
                    // the rows come from the per-item table in registers.
                    const int c = lane;                   // KB == 256: 32 chunks per row
                    const int64_t k = (int64_t)kb * KB + c * 8;
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        const int row = __shfl_sync(0xFFFFFFFFu, gather_row[t >> 5], t & 31);
                        const bool in = row >= 0 && k < p.K;
                        const uint16_t *src = in ? p.A + (int64_t)row * p.K + k : p.A;
                        const uint32_t dst = x_stage(s) + (c >> 3) * L::kXSub + t * 128 +
                                             ((((uint32_t)c & 7u) ^ ((uint32_t)t & 7u)) << 4);
                        cp_async_16(dst, src, in ? 16u : 0u);
                    }
                    cp_async_mbar_arrive(full_bar(s));
                }
            }
        }
        // Drain: wait (bounded) until the loads this warp issued have landed.
        if (lane == 0) {
            const uint32_t first = it > (uint32_t)NSTAGE ? it - NSTAGE : 0u;
            for (uint32_t j = first; j < it; ++j) drain_wait(full_bar(j % NSTAGE), (j / NSTAGE) & 1u);
        }
    };
    // grp: dequant group in [0, NDQ)
    auto role_dequant = [&](const uint32_t grp) {
        // --------------------------------------------------------- dequant
        // NDQ groups of 4 warps, one warp per TMEM lane quarter.  Group g takes
        // every NDQ-th k-block of the CTA's work in full, so one group's barrier
        // waits and shared-memory latency overlap another group's arithmetic.
        // A thread owns one A row (TMEM lane) and unpacks its G chunks (a chunk =
        // 16 bytes of the row = 4 packed words = one group of 32 codes).
        constexpr int G = KB / 32;
        static_assert(G % 2 == 0, "chunks are stored in pairs (32 TMEM columns)");
        const int q4 = warp & 3;                    // TMEM lane quarter of this warp
        const int lrow = q4 * 32 + lane;            // A row of this thread
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int64_t gpr = p.K / 32;               // groups per row
        uint32_t it = 0;
        bool ok = true;
        ItemIter I = make_iter(p, num_items);
        int rt, tt, kb0, kb1;
        while (ok && next_item(I, p, rt, tt, kb0, kb1)) {
            const int64_t row = (int64_t)rt * R + lrow;
            const bool valid = lrow < R && row < p.N;
            const uint16_t *srow = nullptr;
            if (KB != 256 && FP4 == 0 && valid) {
                int64_t base = row * gpr;
                if (MOE) base += (int64_t)__ldg(p.expert_ids + tt / p.moe_sub) * p.N * gpr;
                srow = p.S + base;
            }
            const uint8_t *zrow = (ZP && srow != nullptr) ? p.Z + (srow - p.S) : nullptr;
            if (ZP && KB == 256 && valid) zrow = p.Z + row * gpr;
            // FP4: the row's scale bytes, one per 32 (MX) or 16 (NV) codes
            constexpr int kFpg = FP4 == 2 ? 4 : 2;       // scale bytes per k-block
            const int64_t fgpr = (FP4 == 2) ? p.K / 16 : gpr;
            const uint8_t *frow = (FP4 != 0 && valid) ? p.Z + row * fgpr : nullptr;
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                if (it % NDQ != grp) continue;
                const int s = it % NSTAGE;
                const int a = it % NASTAGE;
                if constexpr (kQdx) {
                    // QAT input gradient: warp q4 takes output rows (K) 32 q4 ..
                    // 32 q4 + 31 of the tile, lane the contraction rows n, n + 1
                    // (n = 2 lane) of the k-block: the two groups of 32 go through
                    // the exact group QDQ, and the results are written transposed,
                    // as the K-major A tile [128 K rows][64 N] (128-byte swizzle)
                    if (!warp_wait(full_bar(s), (it / NSTAGE) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t src = w_stage(s) + (uint32_t)((q4 >> 1) * (L::kWBytes / 2));
                    uint32_t v[2][16], o[2][16];
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint4 x = lds128(
                                src + swz((uint32_t)((2 * lane + h) * 128 + ((q4 & 1) * 4 + c) * 16),
                                          128));
                            v[h][4 * c] = x.x;
                            v[h][4 * c + 1] = x.y;
                            v[h][4 * c + 2] = x.z;
                            v[h][4 * c + 3] = x.w;
                        }
#pragma unroll
                    for (int h = 0; h < 2; ++h) qdq::fake_quant_group(v[h], o[h]);
                    if (!warp_wait(aslot_free_bar(it), aslot_free_parity(it), abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = a_smem(a);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t k0 = (uint32_t)(32 * q4 + 2 * i);
                        sts32(dst + swz(k0 * 128u + 4u * (uint32_t)lane, 128),
                              __byte_perm(o[0][i], o[1][i], 0x5410));
                        sts32(dst + swz((k0 + 1u) * 128u + 4u * (uint32_t)lane, 128),
                              __byte_perm(o[0][i], o[1][i], 0x7632));
                    }
                    fence_proxy_async_smem();       // generic writes -> tensor-core reads
                    mbar_arrive(afull_bar(a));
                    continue;
                }
                if constexpr (kQin) {
                    // QAT forward, in place: the row's 64 BF16 weights (two groups
                    // of 32, one 128-byte swizzled line of the stage) go through
                    // the exact group QDQ and are written back where they were;
                    // the line is this thread's alone, and the stage is reused
                    // only after the MMAs that read it complete
                    if (!warp_wait(full_bar(s), (it / NSTAGE) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint32_t v[2][16], o[2][16];
                    uint32_t addr[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        addr[c] = w_stage(s) + swz((uint32_t)(lrow * 128 + c * 16), 128);
                        const uint4 x = lds128(addr[c]);
                        v[c >> 2][4 * (c & 3)] = x.x;
                        v[c >> 2][4 * (c & 3) + 1] = x.y;
                        v[c >> 2][4 * (c & 3) + 2] = x.z;
                        v[c >> 2][4 * (c & 3) + 3] = x.w;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) qdq::fake_quant_group(v[h], o[h]);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        sts128(addr[c], make_uint4(o[c >> 2][4 * (c & 3)], o[c >> 2][4 * (c & 3) + 1],
                                                   o[c >> 2][4 * (c & 3) + 2],
                                                   o[c >> 2][4 * (c & 3) + 3]));
                    fence_proxy_async_smem();       // generic writes -> tensor-core reads
                    mbar_arrive(afull_bar(a));
                    continue;
                }
                if constexpr (QAT == 1) {
                    // QAT forward: the row's 64 BF16 weights (two groups of 32,
                    // 128-byte swizzled line) go through the exact group QDQ of the
                    // quantizers, straight into this k-block's A columns
                    if (!warp_wait(full_bar(s), (it / NSTAGE) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint32_t v[2][16], o[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 x = lds128(w_stage(s) + swz((uint32_t)(lrow * 128 + c * 16), 128));
                        v[c >> 2][4 * (c & 3)] = x.x;
                        v[c >> 2][4 * (c & 3) + 1] = x.y;
                        v[c >> 2][4 * (c & 3) + 2] = x.z;
                        v[c >> 2][4 * (c & 3) + 3] = x.w;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t og[16];
                        qdq::fake_quant_group(v[h], og);
#pragma unroll
                        for (int z = 0; z < 16; ++z) o[16 * h + z] = og[z];
                    }
                    if (!warp_wait(aslot_free_bar(it), aslot_free_parity(it), abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    tmem_st_x32(tmem_base + lane_addr + (uint32_t)(kABase + a * kAStageCols), o);
                    tmem_wait_st();
                    tc_fence_before_sync();
                    mbar_arrive(afull_bar(a));
                    continue;
                }
                static_assert(KB == 256 || G == 2, "direct-load scales: one chunk pair per k-block");
                uint32_t sc[G] = {}, zb[G] = {};
                float fs[kFpg];
                uint4 kbytes = make_uint4(0u, 0u, 0u, 0u);     // kByteScales: the k-block's bytes
                if constexpr (kByteScales) {
                    const uint8_t *src = ZP ? zrow : frow;
                    if (src != nullptr) {
                        if (FP4 == 2) {
                            kbytes = __ldg(reinterpret_cast<const uint4 *>(src) + kb);
                        } else {
                            const uint2 b8 = __ldg(reinterpret_cast<const uint2 *>(src) + kb);
                            kbytes.x = b8.x;
                            kbytes.y = b8.y;
                        }
                    }
                } else if constexpr (FP4 != 0) {
                    // the k-block's FP4 group scales as FP32 (exact conversions)
#pragma unroll
                    for (int j = 0; j < kFpg; ++j) {
                        const int64_t gi = (int64_t)kb * kFpg + j;
                        const uint32_t b = (frow != nullptr && gi < fgpr) ? __ldg(frow + gi) : 0u;
                        fs[j] = FP4 == 1 ? e8m0_to_f32(b) : e4m3_to_f32(b);
                    }
                } else if (KB != 256) {
                    // scales (and zero points) of this k-block (direct loads when the
                    // tile has no TMA scales)
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const int64_t gi = (int64_t)kb * G + j;
                        const uint16_t v = (srow != nullptr && gi < gpr) ? __ldg(srow + gi) : 0;
                        sc[j] = bf16x2_splat(v);
                        if (ZP)
                            zb[j] = zp_bias2((zrow != nullptr && gi < gpr) ? __ldg(zrow + gi) : 0u);
                    }
                }
                if (!warp_wait(full_bar(s), (it / NSTAGE) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                // The row's 16-byte chunks (and, with TMA-loaded scales, their two
                // scales) are read one pair ahead of their use.  The pair loop stays
                // rolled: one compact body run G / 2 times stays in the instruction
                // cache, where the unrolled k-block would be refetched every time.
                auto load_pair = [&](int j, uint4 (&w)[2]) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj)
                        w[jj] = lds128(w_stage(s) +
                                       swz((uint32_t)(lrow * (KB / 2) + (j + jj) * 16), KB / 2));
                };
                auto load_scales = [&](int j) -> uint32_t {
                    return (KB == 256 && FP4 == 0) ? lds32(s_stage(s) + lrow * 16 + j * 2) : 0u;
                };
                // byte b of the k-block's direct-loaded bytes
                auto kbyte = [&](int b) -> uint32_t {
                    const uint32_t wv = (b >> 2) == 0 ? kbytes.x
                                      : (b >> 2) == 1 ? kbytes.y
                                      : (b >> 2) == 2 ? kbytes.z : kbytes.w;
                    return (wv >> (8 * (b & 3))) & 0xFFu;
                };
                // Two chunks (8 packed words) become 32 TMEM columns, 2 BF16 per column.
                auto unpack_pair = [&](const uint4 (&w)[2], uint32_t s_pair, uint32_t (&o)[32],
                                       int jpair) {
                    uint32_t scp[2];
                    if (KB == 256) {
                        scp[0] = bf16x2_splat((uint16_t)(s_pair & 0xFFFFu));
                        scp[1] = bf16x2_splat((uint16_t)(s_pair >> 16));
                    } else {
                        scp[0] = sc[0];     // G == 2: a single pair
                        scp[1] = sc[1];
                    }
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const uint32_t ws[4] = {w[jj].x, w[jj].y, w[jj].z, w[jj].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t t4[4];
                            const int c = jpair + jj;           // chunk of the k-block
                            if (kByteScales && FP4 == 1)
                                dequant_word_mxfp4(ws[q], e8m0_to_f32(kbyte(c)), t4);
                            else if (kByteScales && FP4 == 2)
                                dequant_word_nvfp4(ws[q], e4m3_to_f32(kbyte(2 * c + (q >> 1))),
                                                   p.fp4_g, t4);
                            else if (kByteScales && ZP)
                                dequant_word_k8perm_zp(ws[q], scp[jj], zp_bias2(kbyte(c)), t4);
                            else if (kXPerm) dequant_word_k8perm(ws[q], scp[jj], t4);
                            else if (FP4 == 1) dequant_word_mxfp4(ws[q], fs[jj], t4);
                            else if (FP4 == 2)
                                dequant_word_nvfp4(ws[q], fs[(2 * jj + (q >> 1)) % kFpg], p.fp4_g,
                                                   t4);
                            else if (ZP) dequant_word_zp(ws[q], scp[jj], zb[jj], t4);
                            else dequant_word(ws[q], scp[jj], t4);
#pragma unroll
                            for (int z = 0; z < 4; ++z) o[jj * 16 + q * 4 + z] = t4[z];
                        }
                    }
                };
                // The first pair is unpacked before the A slot is known to be free,
                // so the wait for the slot overlaps that arithmetic; each later
                // pair is loaded and unpacked while the previous one is stored.
                // Two output buffers alternate, so unpacking a pair never has to
                // wait for the store of the previous pair to read its registers.
                uint4 cur[2];
                load_pair(0, cur);
                uint32_t o[2][32];
                unpack_pair(cur, load_scales(0), o[0], 0);
                if (!warp_wait(aslot_free_bar(it), aslot_free_parity(it), abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t a_col = tmem_base + lane_addr + (uint32_t)(kABase + a * kAStageCols);
                constexpr int kPairs = G / 2;
#pragma unroll
                for (int jp = 0; jp < kPairs; ++jp) {
                    const int j = 2 * jp;
                    uint32_t s_nxt = 0;
                    if (jp + 1 < kPairs) {
                        load_pair(j + 2, cur);
                        s_nxt = load_scales(j + 2);
                    }
                    tmem_st_x32(a_col + (uint32_t)(j * 16), o[jp & 1]);
                    if (jp + 1 < kPairs) unpack_pair(cur, s_nxt, o[(jp + 1) & 1], j + 2);
                }
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(afull_bar(a));
            }
        }
    };
    // pw: index of the activation-reorder warp
    auto role_perm = [&](const int pw) {
        // ------------------------------------------------ activation reorder
        // 256-wide k-blocks: the dequant warps leave codes (j, j + 4) of a packed
        // word in one register pair (dequant_word_k8perm), so every 16-byte
        // activation chunk [x0..x7] of the stage is rewritten in place as
        // [x0, x4, x1, x5, x2, x6, x3, x7].  These warps issue no asynchronous
        // copies or MMAs, so their proxy fence waits only for their own stores.
        uint32_t it = 0;
        bool ok = true;
        ItemIter I = make_iter(p, num_items);
        int rt, tt, kb0, kb1;
        while (ok && next_item(I, p, rt, tt, kb0, kb1)) {
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % NSTAGE;
                if (!warp_wait(full_bar(s), (it / NSTAGE) & 1u, abort_flag, kSleepAhead)) {
                    ok = false;
                    break;
                }
                constexpr int kChunks = MT * (KB / 8);
                // batches of 8 chunks per thread: all loads first, so their
                // latencies overlap
                constexpr int kBatch = 8;
                constexpr int kStride = 32 * (kPermWarps > 0 ? kPermWarps : 1);
                static_assert(kChunks % (kStride * kBatch) == 0, "whole batches");
#pragma unroll 1
                for (int c0 = pw * 32 + lane; FP4 == 0 && c0 < kChunks; c0 += kStride * kBatch) {
                    uint32_t addr[kBatch];
                    uint4 v[kBatch];
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) {
                        const int ci = c0 + b * kStride;
                        const int t = ci / (KB / 8), c = ci % (KB / 8);
                        addr[b] = x_stage(s) + (c >> 3) * L::kXSub + t * 128 +
                                  ((((uint32_t)c & 7u) ^ ((uint32_t)t & 7u)) << 4);
                        v[b] = lds128(addr[b]);
                    }
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) sts128(addr[b], permute_chunk8(v[b]));
                }
                fence_proxy_async_smem();   // generic writes -> tensor-core reads
                // Join the dequant group's arrival on the A slot's "full" barrier.
                // Waiting for the slot to be free first keeps this arrival in the
                // slot's current phase (these warps may run ahead of the dequant).
                const int a = it % NASTAGE;
                if (!warp_wait(aslot_free_bar(it), aslot_free_parity(it), abort_flag, kSleepAhead)) {
                    ok = false;
                    break;
                }
                mbar_arrive(afull_bar(a));
            }
        }
    };
    // kIss: std::true_type for an MMA issuer (index ji), std::false_type for an
    // epilogue warp; each instantiation keeps only its own role's code
    auto role_mma = [&](auto kIss, const int ji) {
        // ------------------------------------------------- MMA + epilogue
        // four epilogue warps (one per TMEM lane quarter), then NSPLIT MMA issuers:
        // the epilogue of one work item overlaps the MMAs of the next
        constexpr bool issuer = decltype(kIss)::value;
        const int q4 = warp & 3;
        const int lrow = q4 * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        uint32_t it = 0, acc_it = 0;
        uint32_t xchg_count = 0;                    // SiLU*up hand-overs so far
        bool ok = true;
        ItemIter I = make_iter(p, num_items);
        int rt, tt, kb0, kb1;
        for (; ok && next_item(I, p, rt, tt, kb0, kb1); ++acc_it) {
            const int d = acc_it % NACC;
            if constexpr (issuer) {
                if (!warp_wait(accempty_bar(d), ((acc_it / NACC) & 1u) ^ 1u, abort_flag, kSleepAhead)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem =
                    tmem_base + (uint32_t)(d * kAccCols + (SPLITN ? ji * kNPer : ji * MT));
                // Lane 0 alone polls and issues: a warp-wide wait adds a vote to
                // every poll, and each poll sits on the issue path between two
                // k-blocks' MMAs.  The issuer waits only for the A slot: the
                // threads that arrive on it (the dequant group, plus the
                // activation-reorder warps with 256-wide k-blocks) each waited
                // for the stage's loads first, so the acquire of the A slot's
                // phase also orders the loaded tiles before these MMAs.
                if (lane == 0) {
                    for (int kb = kb0; kb < kb1; ++kb, ++it) {
                        const int s = it % NSTAGE;
                        const int a = it % NASTAGE;
                        if (!mbar_wait_spin(afull_bar(a), (it / NASTAGE) & 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        if (MOE) fence_proxy_async_smem();   // cp.async (generic proxy) -> MMA
                        const uint32_t a_tmem = tmem_base + (uint32_t)(kABase + a * kAStageCols);
                        // SPLITN: this issuer's tokens start kNPer rows (128 B each,
                        // whole 1024-byte swizzle atoms) into the activation tile
                        constexpr int kU0Step = SPLITN ? 1 : NSPLIT;
                        const uint32_t xrow = SPLITN ? (uint32_t)(ji * kNPer * 128) : 0u;
#pragma unroll
                        for (int u = SPLITN ? 0 : ji; u < KB / 16; u += kU0Step) {
                            const uint32_t baddr =
                                x_stage(s) + (u >> 2) * L::kXSub + (u & 3) * 32 + xrow;
                            const uint32_t acc_flag = (kb > kb0 || u >= kU0Step) ? 1u : 0u;
                            if (kQdx)
                                tc_mma_ss(d_tmem, smem_desc_k_sw128(a_smem(a) + (u & 3) * 32),
                                          smem_desc_k_sw128(baddr), kIdesc, acc_flag);
                            else if (kQin)
                                tc_mma_ss(d_tmem, smem_desc_k_sw128(w_stage(s) + (u & 3) * 32),
                                          smem_desc_k_sw128(baddr), kIdesc, acc_flag);
                            else
                                tc_mma_ts(d_tmem, a_tmem + u * 8, smem_desc_k_sw128(baddr), kIdesc,
                                          acc_flag);
                        }
                        tc_commit(empty_bar(s));
                        if (!kOneRelease) tc_commit(aempty_bar(a));
                    }
                } else {
                    it += (uint32_t)(kb1 - kb0);
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
                it = __shfl_sync(0xFFFFFFFFu, it, 0);
                if (!ok) break;
                if (lane == 0) tc_commit(accfull_bar(d));
                __syncwarp();
                continue;                           // issuers do no epilogue
            }
            // epilogue of this lane quarter: sum the NSPLIT accumulators in order
            if (!warp_wait(accfull_bar(d), (acc_it / NACC) & 1u, abort_flag, kSleepLong)) break;
            tc_fence_after_sync();
            const int64_t row = (int64_t)rt * R + lrow;
            const bool valid = lrow < R && row < p.N;
            // split item: this CTA holds only part of the row tile's K range
            const bool partial = p.split && !(kb0 == 0 && kb1 == p.num_kb);
            int contrib = 1, my_idx = 0;
            float *my_part = nullptr;
            if (partial) {
                const int c_first = unit_owner((uint32_t)rt * (uint32_t)p.num_kb, p);
                const int c_last = unit_owner((uint32_t)rt * (uint32_t)p.num_kb + (uint32_t)p.num_kb - 1u, p);
                contrib = c_last - c_first + 1;
                my_idx = blockIdx.x - c_first;
                my_part = p.ws_part + (((int64_t)rt * p.max_contrib + my_idx) * 128 + lrow) * MT;
            }
            unsigned int *cnt = partial ? p.ws_cnt + (int64_t)rt * 4 + q4 : nullptr;
            // 16-column tiles: when every other contributor has already parked its
            // partial (the usual case for the CTA's last item), this warp sums
            // them with its own, still in registers, without parking or counting.
            constexpr bool kDirect = MT == 16 && !MOE;
            bool last_now = false;
            uint32_t own[16];
            if (kDirect && partial) {
                unsigned int seen = 0;
                if (lane == 0) seen = ld_acquire_gpu(cnt);
                seen = __shfl_sync(0xFFFFFFFFu, seen, 0);
                __syncwarp();
                last_now = seen == (unsigned int)(contrib - 1);
            }
#pragma unroll 1
            for (int c0 = 0; c0 < MT; c0 += 16) {
                // all NSPLIT accumulator loads in flight, one wait, then the sum in
                // accumulator order (two at a time, to bound the registers)
                uint32_t v[16];
                constexpr int kLd = kAccSets < 2 ? kAccSets : 2;
#pragma unroll
                for (int sp0 = 0; sp0 < kAccSets; sp0 += kLd) {
                    uint32_t w2[kLd][16];
#pragma unroll
                    for (int sp = 0; sp < kLd; ++sp)
                        tmem_ld_x16(tmem_base + lane_addr +
                                        (uint32_t)(d * kAccCols + (sp0 + sp) * MT + c0),
                                    w2[sp]);
                    tmem_wait_ld();
#pragma unroll
                    for (int sp = 0; sp < kLd; ++sp)
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            v[jj] = (sp0 + sp == 0)
                                        ? w2[0][jj]
                                        : __float_as_uint(__uint_as_float(v[jj]) +
                                                          __uint_as_float(w2[sp][jj]));
                }
                if (partial) {
                    if (kDirect && last_now) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) own[jj] = v[jj];
                        continue;
                    }
                    // park this CTA's partial sums (fp32) for the row tile's last arriver
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        __stcg(reinterpret_cast<float4 *>(my_part + c0) + q,
                               make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                           __uint_as_float(v[4 * q + 2]),
                                           __uint_as_float(v[4 * q + 3])));
                    continue;
                }
                if (MOE && p.silu_inter > 0) {
                    // h = bf16(silu(g) * u): lane quarters 0-1 hold the gate rows,
                    // 2-3 the up rows of the same 64 output columns; the up values
                    // cross through shared memory (bounded mbarrier hand-over)
                    const uint32_t xc = xchg_count++;
                    float *xrow = xchg + ((q4 & 1) * 32 + lane) * 16;
                    if (q4 >= 2) {
                        if (xc > 0 && !warp_wait(smem_u32(&xchg_bar[1]), (xc - 1) & 1u,
                                                 abort_flag, kPollSleepNs))
                            break;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            reinterpret_cast<float4 *>(xrow)[q] = make_float4(
                                __uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&xchg_bar[0]));
                    } else {
                        if (!warp_wait(smem_u32(&xchg_bar[0]), xc & 1u, abort_flag, kPollSleepNs))
                            break;
                        const int64_t hcol = (int64_t)rt * 64 + q4 * 32 + lane;
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const float g = __uint_as_float(v[jj]);
                            const float u = xrow[jj];
                            const int slot = __ldg(p.sorted_ids + (int64_t)tt * MT + c0 + jj);
                            if (hcol < p.silu_inter && slot >= 0 && slot < p.num_slots) {
                                const __nv_bfloat16 h =
                                    __float2bfloat16_rn((g / (1.0f + expf(-g))) * u);
                                p.Y[(int64_t)slot * p.silu_inter + hcol] =
                                    *reinterpret_cast<const uint16_t *>(&h);
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&xchg_bar[1]));
                    }
                    continue;
                }
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int tok = c0 + jj;
                    int64_t out_row;
                    if (MOE) {
                        const int slot = __ldg(p.sorted_ids + (int64_t)tt * MT + tok);
                        out_row = (slot >= 0 && slot < p.num_slots) ? slot : -1;
                    } else {
                        const int64_t m = (int64_t)tt * MT + tok;
                        out_row = (m < p.M) ? m : -1;
                    }
                    if (valid && out_row >= 0) {
                        const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[jj]));
                        p.Y[out_row * p.N + row] = *reinterpret_cast<const uint16_t *>(&h);
                    }
                }
                if (MOE && p.comb_out != nullptr) {
                    // Fused combine.  Lane j < 16 counts column c0 + j's slot in
                    // for its token (this warp's 32 rows of the row tile); the
                    // lane that brings a token's count to topk has seen every
                    // slot row of it written, and the warp then sums them in
                    // ascending k -- the arithmetic of w4_moe_combine, so the
                    // result does not depend on which work item came last.
                    // One GPU-scope fence by lane 0 after __syncwarp releases all
                    // lanes' C stores before the (relaxed) count updates; a
                    // warp that sees a count complete fences again (acquire)
                    // before reading the other slot rows.
                    __syncwarp();
                    if (lane == 0) __threadfence();
                    __syncwarp();
                    int slot = -1;
                    if (lane < 16) {
                        slot = __ldg(p.sorted_ids + (int64_t)tt * MT + c0 + lane);
                        if (slot < 0 || slot >= p.num_slots) slot = -1;
                    }
                    bool last = false;
                    if (slot >= 0) {
                        unsigned int *cnt_t =
                            p.comb_cnt + ((int64_t)(slot / p.topk) * p.n_row_tiles + rt) * 4 + q4;
                        last = atomicAdd(cnt_t, 1u) == (unsigned int)(p.topk - 1);
                    }
                    unsigned int todo = __ballot_sync(0xFFFFFFFFu, last);
                    if (todo != 0u) __threadfence();
                    __syncwarp();
                    while (todo != 0u) {
                        const int j = __ffs(todo) - 1;
                        todo &= todo - 1u;
                        const int64_t t = __shfl_sync(0xFFFFFFFFu, slot, j) / p.topk;
                        if (valid) {
                            float acc = 0.0f;
                            for (int k = 0; k < p.topk; ++k) {
                                const float wk = __ldg(p.comb_w + t * p.topk + k);
                                const uint16_t d = __ldcg(p.Y + (t * p.topk + k) * p.N + row);
                                acc = __fadd_rn(acc, __fmul_rn(wk, __uint_as_float((uint32_t)d << 16)));
                            }
                            const __nv_bfloat16 h = __float2bfloat16_rn(acc);
                            p.comb_out[t * p.N + row] = *reinterpret_cast<const uint16_t *>(&h);
                        }
                        if (lane == j)
                            p.comb_cnt[(t * p.n_row_tiles + rt) * 4 + q4] = 0u;   // next call
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(accempty_bar(d));
            if (kDirect && partial && last_now) {
                // Sum in ascending K order: the parked partials, with this CTA's own
                // values in its place, then write Y and reset the counter.
                const float *base = p.ws_part + ((int64_t)rt * p.max_contrib * 128 + lrow) * MT;
                float acc[16];
                for (int ci = 0; ci < contrib; ++ci) {
                    if (ci == my_idx) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            acc[jj] = ci == 0 ? __uint_as_float(own[jj])
                                              : acc[jj] + __uint_as_float(own[jj]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 f = __ldcg(
                                reinterpret_cast<const float4 *>(base + (int64_t)ci * 128 * MT) + q);
                            const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                acc[4 * q + e] = ci == 0 ? fv[e] : acc[4 * q + e] + fv[e];
                        }
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    if (valid && jj < p.M) {
                        const __nv_bfloat16 h = __float2bfloat16_rn(acc[jj]);
                        p.Y[(int64_t)jj * p.N + row] = *reinterpret_cast<const uint16_t *>(&h);
                    }
                }
                if (lane == 0) *cnt = 0u;           // ready for the next call
            } else if (partial) {
                // The last of the row tile's contributing warps (per lane quarter)
                // adds all partials in ascending K order and writes Y.
                // __syncwarp orders the lanes' partial stores before lane 0's
                // count update, whose release makes them visible GPU-wide; the
                // acquire side of the same update, then __syncwarp, orders the
                // last arriver's reads of the other partials after it.
                __syncwarp();
                unsigned int old = 0;
                if (lane == 0) old = atom_add_acq_rel_gpu(cnt, 1u);
                old = __shfl_sync(0xFFFFFFFFu, old, 0);
                if (old == (unsigned int)(contrib - 1)) {
                    __syncwarp();
                    const float *base =
                        p.ws_part + ((int64_t)rt * p.max_contrib * 128 + lrow) * MT;
                    // 16 columns at a time, contributions in ascending K order: the
                    // four loads of one contribution are in flight together
#pragma unroll 1
                    for (int c0 = 0; c0 < MT; c0 += 16) {
                        float4 acc[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            acc[q] = __ldcg(reinterpret_cast<const float4 *>(base + c0) + q);
                        for (int ci = 1; ci < contrib; ++ci) {
                            float4 t[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                t[q] = __ldcg(reinterpret_cast<const float4 *>(
                                                  base + (int64_t)ci * 128 * MT + c0) + q);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                acc[q].x += t[q].x;
                                acc[q].y += t[q].y;
                                acc[q].z += t[q].z;
                                acc[q].w += t[q].w;
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float av[4] = {acc[q].x, acc[q].y, acc[q].z, acc[q].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int64_t m = c0 + 4 * q + e;
                                if (valid && m < p.M) {
                                    const __nv_bfloat16 h = __float2bfloat16_rn(av[e]);
                                    p.Y[m * p.N + row] = *reinterpret_cast<const uint16_t *>(&h);
                                }
                            }
                        }
                    }
                    if (lane == 0) *cnt = 0u;       // ready for the next call
                }
            }
        }
        // all MMAs issued by this warp complete before TMEM is released
        if constexpr (issuer) {
            if (lane == 0) {
                tc_commit(mmadone_bar);
                drain_wait(mmadone_bar, 0u);
            }
            __syncwarp();
        }
    };

    if constexpr (WGL) {
        // Each warpgroup first resizes its register file (every warp of the
        // warpgroup executes its setmaxnreg), so the compiler fits each role
        // into that count.
        const int wg = warp >> 2;
        constexpr int kLaunch = launch_regs_wgl(NDQ);
        if (wg == kWgLoad) {
            reg_set<kRegsLoad, kLaunch>();
            if (warp == kAllocWarp) role_loads();
            else if (warp - kAllocWarp <= kPermWarps) role_perm(warp - kAllocWarp - 1);
        } else if (wg < NDQ) {
            reg_set<dequant_regs_wgl(NDQ), kLaunch>();
            role_dequant((uint32_t)wg);
        } else if (wg == NDQ) {
            reg_set<kRegsEpi, kLaunch>();
            role_mma(std::false_type{}, -1);
        } else {
            reg_set<kRegsIssue, kLaunch>();
            const int ji = warp - 4 * (NDQ + 1);
            if (ji < NSPLIT) role_mma(std::true_type{}, ji);
        }
    } else {
        if (warp == 0) role_loads();
        else if (warp < 1 + kDqWarps) role_dequant((uint32_t)(warp - 1) >> 2);
        else if (warp < kEpiWarp0) role_perm(warp - 1 - kDqWarps);
        else if (warp < kEpiWarp0 + 4) role_mma(std::false_type{}, -1);
        else role_mma(std::true_type{}, warp - kEpiWarp0 - 4);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kAllocWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int KB, int MT, int NSTAGE, int NACC, int NASTAGE, int NSPLIT, int NDQ, bool MOE,
          bool WGL = false, int QAT = 0, bool ZP = false, bool SPLITN = false, int FP4 = 0>
w4_status launch_cfg(const CUtensorMap &tw, const CUtensorMap &ts, const CUtensorMap &tx,
                     const GemmParams &p, int num_items_max, cudaStream_t stream) {
    using L = Layout<KB, MT, NSTAGE, NACC, NASTAGE, (SPLITN ? 1 : NSPLIT), (QAT != 0), (QAT == 2),
                     (QAT <= 1)>;
    auto kern =
        w4a16_tc_kernel<KB, MT, NSTAGE, NACC, NASTAGE, NSPLIT, NDQ, MOE, WGL, QAT, ZP, SPLITN, FP4>;
    // At least half of the SM's shared memory, so one CTA (and one TMEM
    // allocation of 512 columns) per SM.
    const int smem = std::max(L::kAlloc, 120 * 1024);
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return w4host::launch_status();
        configured = true;
    }
    if (WGL) {
        // setmaxnreg draws on the registers the CTA was launched with: refuse to
        // launch (rather than wait forever) if the build gave fewer than the
        // split needs.
        static int regs_built = -1;
        if (regs_built < 0) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return w4host::launch_status();
            regs_built = fa.numRegs;
        }
        if (regs_built * gemm_threads(NDQ, KB, NSPLIT, WGL) < 128 * split_regs_wgl(NDQ))
            return W4_ERR_UNSUPPORTED;
    }
    const int grid = std::max(1, std::min(num_items_max, w4host::num_sms()));
    const cudaError_t e = w4host::launch_pdl(kern, dim3(grid), dim3(gemm_threads(NDQ, KB, NSPLIT, WGL)),
                                             (size_t)smem, stream, tw, ts, tx, p);
    if (e != cudaSuccess) {
        w4host::set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    return w4host::launch_status();
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *ptr,
              const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
              CUtensorMapSwizzle sw) {
    return w4host::encode_tiled(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides,
                                box, sw) == CUDA_SUCCESS;
}

int ceil_div_i(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace
}  // namespace w4

using namespace w4;

namespace w4 {
namespace {

// Plan of the stream-K split for a decode-shaped GEMM (M <= 64, K % 256 == 0)
// on `sms` CTAs; returns false when the split does not apply.
struct SplitPlan {
    int n_rt, nkb, ctas, max_contrib, mt;
    size_t cnt_bytes, part_bytes;
};

// The arrival counters sit in a fixed region at the start of the workspace,
// large enough for every row-tile count the split accepts, and the partial
// sums after it: a call's partials (left in place) can then never lie where a
// later call on the same workspace, with more row tiles, expects zeroed
// counters.
constexpr size_t kSplitCntBytes = 4096;
constexpr int64_t kSplitMaxRowTiles = kSplitCntBytes / (4 * sizeof(unsigned int));

bool plan_split(int64_t M, int64_t N, int64_t K, int sms, SplitPlan *sp) {
    if (M > 64 || (K % 256) != 0) return false;
    const int64_t n_rt = (N + 127) / 128, nkb = K / 256;
    if (n_rt >= sms || nkb < 2 || n_rt > kSplitMaxRowTiles) return false;
    const int64_t units = n_rt * nkb;
    const int ctas = (int)std::min<int64_t>(sms, units);
    if (units * (ctas + 1) >= ((int64_t)1 << 32)) return false;   // device math is 32-bit
    auto owner = [&](int64_t x) { return (int)(((x + 1) * ctas - 1) / units); };
    int mc = 1;
    for (int64_t rt = 0; rt < n_rt; ++rt)
        mc = std::max(mc, owner(rt * nkb + nkb - 1) - owner(rt * nkb) + 1);
    sp->n_rt = (int)n_rt;
    sp->nkb = (int)nkb;
    sp->ctas = ctas;
    sp->max_contrib = mc;
    sp->mt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    sp->cnt_bytes = kSplitCntBytes;
    sp->part_bytes = (size_t)n_rt * mc * 128 * sp->mt * sizeof(float);
    return true;
}

}  // namespace
}  // namespace w4

namespace w4 {
namespace {

// One warp waits, with the GEMM's bounded wait, for a phase of an mbarrier
// that nothing completes: the wait gives up after limit_ns, records the
// timeout in the device status word and the kernel returns.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1u);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    mbar_wait(smem_u32(&bar), 0u, &abort_flag, kPollSleepNs, limit_ns);
}

}  // namespace
}  // namespace w4

extern "C" w4_status w4_wait_selftest(uint32_t limit_us, void *stream) {
    if (limit_us == 0 || limit_us > 1000000u) return W4_ERR_INVALID_ARG;
    w4::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(1000ull * limit_us);
    return w4host::launch_status();
}

cudaError_t w4host::gemm_device_status(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, w4::g_device_status, sizeof *flag);
    if (e == cudaSuccess && *flag != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(w4::g_device_status, &zero, sizeof zero);
    }
    return e;
}

extern "C" size_t w4a16_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    SplitPlan sp;
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    if (w4host::gemv_supported(M, N, K)) return 0;
    if (!plan_split(M, N, K, w4host::num_sms(), &sp)) return 0;
    return sp.cnt_bytes + sp.part_bytes;
}

extern "C" w4_status w4a16_gemm(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                                w4_bf16 *Y, int64_t M, int64_t N, int64_t K, int group,
                                void *workspace, size_t workspace_bytes, void *stream) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(X) || !w4host::aligned16(Wq) || !w4host::aligned16(S) ||
        !w4host::aligned16(Y))
        return W4_ERR_INVALID_ARG;
    if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    if (N > (1 << 30) || M > (1 << 30) || K > (1 << 24)) return W4_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    // 1..8 activation rows: the warp-level MMA kernel unpacks straight into
    // MMA fragments (w4_gemv.cu), no tensor memory.
    if (w4host::gemv_supported(M, N, K)) {
        const w4_status gs = w4host::gemv_launch(X, Wq, S, Y, M, N, K, stream);
        if (gs != W4_ERR_UNSUPPORTED) return gs;     // else: too many rows per SM, below
    }

    GemmParams p = {};
    p.S = reinterpret_cast<const uint16_t *>(S);
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;

    const int sms = w4host::num_sms();
    const bool wide_k = (K % 256) == 0;
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);

    // X: [M, K] BF16, 64-wide K boxes of MT rows, 128-byte swizzle.
    auto map_x = [&](int mt) {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)mt};
        return make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    };
    auto map_w = [&](int kb, int R) {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        cuuint32_t box[2] = {(cuuint32_t)(kb / 8), (cuuint32_t)R};
        return make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, Wq, dims, strides, box,
                        kb == 256 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B);
    };
    auto map_s = [&](int R) {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 32), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 16)};
        cuuint32_t box[2] = {8u, (cuuint32_t)R};
        return make_map(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, S, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    };

    if (M <= 64 && wide_k) {
        const int mt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
        p.n_tok_tiles = 1;
        p.num_kb = ceil_div_i(K, 256);
        SplitPlan sp;
        int items;
        if (workspace != nullptr && plan_split(M, N, K, sms, &sp) &&
            workspace_bytes >= sp.cnt_bytes + sp.part_bytes) {
            // Decode, stream-K: full 128-row tiles, the (row tile, k-block)
            // units cut evenly over the SMs, partial tiles reduced in a fixed
            // order by the last arriving CTA.
            p.rows_per_tile = 128;
            p.n_row_tiles = sp.n_rt;
            p.split = 1;
            p.units = (int64_t)sp.n_rt * sp.nkb;
            p.ctas = sp.ctas;
            p.max_contrib = sp.max_contrib;
            p.ws_cnt = reinterpret_cast<unsigned int *>(workspace);
            p.ws_part = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) +
                                                  sp.cnt_bytes);
            items = sp.ctas;
            if (!map_x(mt) || !map_w(256, 128) || !map_s(128)) return W4_ERR_CUDA;
        } else {
            // Decode without a workspace: one token tile, N split evenly over
            // the SMs (rows per tile = ceil(N / SMs)).
            int R = std::min<int64_t>(128, std::max<int64_t>(1, ceil_div_i(N, sms)));
            while (R < 128 && ceil_div_i(N, R) > sms) ++R;
            p.rows_per_tile = R;
            p.n_row_tiles = ceil_div_i(N, R);
            items = p.n_row_tiles;
            if (!map_x(mt) || !map_w(256, R) || !map_s(R)) return W4_ERR_CUDA;
        }
        if (mt == 16) return launch_cfg<256, 16, 6, 2, 3, 4, 2, false, true>(tw, ts, tx, p, items, st);
        if (mt == 32) return launch_cfg<256, 32, 6, 2, 2, 4, 2, false, false>(tw, ts, tx, p, items, st);
        return launch_cfg<256, 64, 4, 1, 2, 4, 2, false>(tw, ts, tx, p, items, st);
    }
    // Prefill (and any K that is not a multiple of 256): 128-row tiles,
    // 64-wide K blocks, scales read directly.
    const int mt = M <= 64 ? 64 : 256;
    p.rows_per_tile = 128;
    p.n_row_tiles = ceil_div_i(N, 128);
    p.n_tok_tiles = ceil_div_i(M, mt);
    p.num_kb = ceil_div_i(K, 64);
    if (!map_x(mt) || !map_w(64, 128)) return W4_ERR_CUDA;
    const int64_t items = (int64_t)p.n_row_tiles * p.n_tok_tiles;
    if (items > (1 << 30)) return W4_ERR_UNSUPPORTED;
    if (mt == 64) return launch_cfg<64, 64, 8, 1, 8, 4, 2, false>(tw, ts, tx, p, (int)items, st);
    // two issuers, 128 tokens each (measured: 2-4 % faster than one; four were slower)
    return launch_cfg<64, 256, 6, 1, 6, 2, 2, false, false, false, false, true>(tw, ts, tx, p,
                                                                               (int)items, st);
}

namespace w4 {
namespace {

// Stream-K plan for a QAT GEMM with a single token tile (M <= 256): the
// (128-row tile, 64-wide k-block) units cut evenly over the SMs, as in the
// decode split, when the row tiles alone would leave most SMs idle (fewer than
// half the SMs: measured, the split costs more than it gains above that, e.g.
// the forward at 96 row tiles and 256 tokens).
bool plan_split_qat(int64_t M, int64_t rows, int64_t contraction, int sms, SplitPlan *sp) {
    if (M > 256) return false;
    const int64_t n_rt = (rows + 127) / 128, nkb = (contraction + 63) / 64;
    if (2 * n_rt > sms || nkb < 2 || n_rt > kSplitMaxRowTiles) return false;
    const int64_t units = n_rt * nkb;
    const int ctas = (int)std::min<int64_t>(sms, units);
    if (units * (ctas + 1) >= ((int64_t)1 << 32)) return false;
    auto owner = [&](int64_t x) { return (int)(((x + 1) * ctas - 1) / units); };
    int mc = 1;
    for (int64_t rt = 0; rt < n_rt; ++rt)
        mc = std::max(mc, owner(rt * nkb + nkb - 1) - owner(rt * nkb) + 1);
    sp->n_rt = (int)n_rt;
    sp->nkb = (int)nkb;
    sp->ctas = ctas;
    sp->max_contrib = mc;
    sp->mt = M <= 64 ? 64 : 256;
    sp->cnt_bytes = kSplitCntBytes;
    sp->part_bytes = (size_t)n_rt * mc * 128 * sp->mt * sizeof(float);
    return true;
}

// Applies a QAT split plan to the kernel parameters (false: run unsplit).
bool use_split_qat(GemmParams &p, int64_t M, int64_t rows, int64_t contraction, void *workspace,
                   size_t workspace_bytes, int *items) {
    SplitPlan sp;
    if (workspace == nullptr ||
        !plan_split_qat(M, rows, contraction, w4host::num_sms(), &sp) ||
        workspace_bytes < sp.cnt_bytes + sp.part_bytes)
        return false;
    p.n_row_tiles = sp.n_rt;
    p.split = 1;
    p.units = (int64_t)sp.n_rt * sp.nkb;
    p.ctas = sp.ctas;
    p.max_contrib = sp.max_contrib;
    p.ws_cnt = reinterpret_cast<unsigned int *>(workspace);
    p.ws_part = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + sp.cnt_bytes);
    *items = sp.ctas;
    return true;
}

}  // namespace
}  // namespace w4

extern "C" size_t w4_qat_gemm_workspace_bytes(int64_t M, int64_t rows, int64_t contraction) {
    SplitPlan sp;
    if (M <= 0 || rows <= 0 || contraction <= 0) return 0;
    if (!plan_split_qat(M, rows, contraction, w4host::num_sms(), &sp)) return 0;
    return sp.cnt_bytes + sp.part_bytes;
}

extern "C" w4_status w4_qat_gemm(const w4_bf16 *X, const w4_bf16 *W, w4_bf16 *Y, int64_t M,
                                 int64_t N, int64_t K, int group, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(X) || !w4host::aligned16(W) || !w4host::aligned16(Y))
        return W4_ERR_INVALID_ARG;
    if ((K % 64) != 0) return W4_ERR_UNSUPPORTED;
    if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    if (N > (1 << 30) || M > (1 << 30) || K > (1 << 24)) return W4_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    GemmParams p = {};
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    // more than 64 tokens: 256-token work items with the QDQ written back over
    // the weight tile (A from shared memory), which leaves tensor memory to two
    // accumulator sets, so one item's epilogue overlaps the next item's MMAs
    // (64-token items to fill idle SMs measured slower: each token tile pays
    // the QDQ of every weight tile again)
    const int mt = M <= 64 ? 64 : 256;
    p.rows_per_tile = 128;
    p.n_row_tiles = ceil_div_i(N, 128);
    p.n_tok_tiles = ceil_div_i(M, mt);
    p.num_kb = (int)(K / 64);
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)std::min(mt, 256)};
        if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        // BF16 weights [N, K]: 64-wide K boxes (128-byte lines) of 128 rows
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, 128u};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    if ((int64_t)p.n_row_tiles * p.n_tok_tiles > (1 << 30)) return W4_ERR_UNSUPPORTED;
    int items = p.n_row_tiles * p.n_tok_tiles;
    // one token tile and fewer row tiles than SMs: stream-K over the k-blocks
    use_split_qat(p, M, N, K, workspace, workspace_bytes, &items);
    if (mt == 64)
        return launch_cfg<64, 64, 8, 1, 8, 4, 2, false, false, 1>(tw, ts, tx, p, items, st);
    return launch_cfg<64, 256, 4, 2, 4, 2, 2, false, false, 3, false, true>(tw, ts, tx, p, items,
                                                                           st);
}

extern "C" w4_status w4_qat_gemm_dx(const w4_bf16 *dY, const w4_bf16 *W, w4_bf16 *dX, int64_t M,
                                    int64_t N, int64_t K, int group, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(dY) || !w4host::aligned16(W) || !w4host::aligned16(dX))
        return W4_ERR_INVALID_ARG;
    if ((K % 64) != 0 || (N % 8) != 0) return W4_ERR_UNSUPPORTED;
    if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return W4_ERR_INVALID_ARG;
    if (M == 0) return W4_OK;
    if (N > (1 << 24) || M > (1 << 30) || K > (1 << 30)) return W4_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    if (N == 0) return cudaMemsetAsync(dX, 0, (size_t)M * K * 2, st) == cudaSuccess
                           ? W4_OK : w4host::launch_status();
    // output rows of the kernel = K, contraction = N (64-wide k-blocks), tokens = M
    GemmParams p = {};
    p.Y = reinterpret_cast<uint16_t *>(dX);
    p.M = M;
    p.N = K;
    p.K = N;
    const int mt = M <= 64 ? 64 : 256;
    p.rows_per_tile = 128;
    p.n_row_tiles = ceil_div_i(K, 128);
    p.n_tok_tiles = ceil_div_i(M, mt);
    p.num_kb = ceil_div_i(N, 64);
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);
    {
        // dY [M, N]: 64-wide N boxes of up to 256 tokens
        cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)N * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)std::min(mt, 256)};
        if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dY, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        // W [N, K]: 64 x 64 boxes (128-byte lines along K)
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, 64u};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    if ((int64_t)p.n_row_tiles * p.n_tok_tiles > (1 << 30)) return W4_ERR_UNSUPPORTED;
    int items = p.n_row_tiles * p.n_tok_tiles;
    // one token tile and fewer row tiles than SMs (K = 4096 has only 32):
    // stream-K over the contraction
    use_split_qat(p, M, K, N, workspace, workspace_bytes, &items);
    if (mt == 64)
        return launch_cfg<64, 64, 4, 1, 4, 4, 2, false, false, 2>(tw, ts, tx, p, items, st);
    // two accumulator sets (A is in shared memory), two issuers over the
    // 256 tokens
    return launch_cfg<64, 256, 3, 2, 3, 2, 2, false, false, 2, false, true>(tw, ts, tx, p, items,
                                                                           st);
}

namespace w4 {
namespace {
template <bool ZP, int FP4>
w4_status decode_tiles_bytes(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                             const uint8_t *SB, float g, w4_bf16 *Y, int64_t M, int64_t N,
                             int64_t K, cudaStream_t st);
}  // namespace
}  // namespace w4

extern "C" w4_status w4a16_gemm_zp(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                                   const uint8_t *Z, w4_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                   int group, void *stream) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(X) || !w4host::aligned16(Wq) || !w4host::aligned16(S) ||
        !w4host::aligned16(Y) || Z == nullptr)
        return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    if (N > (1 << 30) || M > (1 << 30) || K > (1 << 24)) return W4_ERR_UNSUPPORTED;
    // 1..8 activation rows: the warp-level MMA kernel (w4_gemv.cu) when K and
    // Z suit its TMA boxes
    if (w4host::gemv_supported(M, N, K)) {
        const w4_status gs = w4host::gemv_launch_zp(X, Wq, S, Z, Y, M, N, K, stream);
        if (gs != W4_ERR_UNSUPPORTED) return gs;
    }
    cudaStream_t st = (cudaStream_t)stream;
    // up to 64 rows: the 256-wide decode tiles, zero points read directly
    if (M <= 64 && (K % 256) == 0 && w4host::aligned16(Z))
        return decode_tiles_bytes<true, 0>(X, Wq, S, Z, 1.0f, Y, M, N, K, st);
    GemmParams p = {};
    p.S = reinterpret_cast<const uint16_t *>(S);
    p.Z = Z;
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    // every M: 128-row tiles, 64-wide K blocks, scales and zero points read
    // directly by the dequant warps
    const int mt = M <= 64 ? 64 : 256;
    p.rows_per_tile = 128;
    p.n_row_tiles = ceil_div_i(N, 128);
    p.n_tok_tiles = ceil_div_i(M, mt);
    p.num_kb = ceil_div_i(K, 64);
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)mt};
        if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        cuuint32_t box[2] = {8u, 128u};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_32B))
            return W4_ERR_CUDA;
    }
    const int64_t items = (int64_t)p.n_row_tiles * p.n_tok_tiles;
    if (items > (1 << 30)) return W4_ERR_UNSUPPORTED;
    if (mt == 64)
        return launch_cfg<64, 64, 8, 1, 8, 4, 2, false, false, false, true>(tw, ts, tx, p,
                                                                           (int)items, st);
    return launch_cfg<64, 256, 6, 1, 6, 2, 2, false, false, false, true, true>(tw, ts, tx, p,
                                                                              (int)items, st);
}

namespace w4 {
namespace {

// Decode-shaped GEMM (9..64 rows, K % 256 == 0) on zero-point groups or FP4
// codes: the 256-wide tensor-memory tiles of w4a16_gemm without a workspace
// (rows split evenly over the SMs, each tile all of K), the byte scales read
// directly by the dequant warps.  S: BF16 scales (zero points only); SB: the
// zero points or FP4 scale bytes.
template <bool ZP, int FP4>
w4_status decode_tiles_bytes(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                             const uint8_t *SB, float g, w4_bf16 *Y, int64_t M, int64_t N,
                             int64_t K, cudaStream_t st) {
    const int sms = w4host::num_sms();
    GemmParams p = {};
    p.S = reinterpret_cast<const uint16_t *>(S);
    p.Z = SB;
    p.fp4_g = g;
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    const int mt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    int R = std::min<int64_t>(128, std::max<int64_t>(1, ceil_div_i(N, sms)));
    while (R < 128 && ceil_div_i(N, R) > sms) ++R;
    p.rows_per_tile = R;
    p.n_row_tiles = ceil_div_i(N, R);
    p.n_tok_tiles = 1;
    p.num_kb = (int)(K / 256);
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)mt};
        if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        cuuint32_t box[2] = {32u, (cuuint32_t)R};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    if (FP4 == 0) {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 32), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 16)};
        cuuint32_t box[2] = {8u, (cuuint32_t)R};
        if (!make_map(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, S, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return W4_ERR_CUDA;
    }
    const int items = p.n_row_tiles;
    if (mt == 16)
        return launch_cfg<256, 16, 6, 2, 3, 4, 2, false, false, 0, ZP, false, FP4>(tw, ts, tx, p,
                                                                                  items, st);
    if (mt == 32)
        return launch_cfg<256, 32, 6, 2, 2, 4, 2, false, false, 0, ZP, false, FP4>(tw, ts, tx, p,
                                                                                  items, st);
    return launch_cfg<256, 64, 4, 1, 2, 4, 2, false, false, 0, ZP, false, FP4>(tw, ts, tx, p, items,
                                                                              st);
}

}  // namespace
}  // namespace w4

namespace w4 {
namespace {

// W4A16 GEMM on FP4 codes (FP4 = 1: MXFP4, 2: NVFP4): the zero-point kernel's
// tiles (128 weight rows x 64-wide k-blocks, scale bytes read directly by the
// dequant warps) with the FP4 unpack in the weight prologue.
template <int FP4>
w4_status gemm_fp4(const w4_bf16 *X, const int32_t *Wq, const uint8_t *SB, float g, w4_bf16 *Y,
                   int64_t M, int64_t N, int64_t K, void *stream) {
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (!w4host::aligned16(X) || !w4host::aligned16(Wq) || !w4host::aligned16(Y) ||
        SB == nullptr)
        return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    if (N > (1 << 30) || M > (1 << 30) || K > (1 << 24)) return W4_ERR_UNSUPPORTED;
    // 1..8 activation rows: the warp-level MMA kernel (w4_gemv.cu) when K and
    // the scale bytes suit its TMA boxes
    if (w4host::gemv_supported(M, N, K)) {
        const w4_status gs = w4host::gemv_launch_fp4(FP4, X, Wq, SB, g, Y, M, N, K, stream);
        if (gs != W4_ERR_UNSUPPORTED) return gs;
    }
    cudaStream_t st = (cudaStream_t)stream;
    // up to 64 rows: the 256-wide decode tiles
    if (M <= 64 && (K % 256) == 0 && w4host::aligned16(SB))
        return decode_tiles_bytes<false, FP4>(X, Wq, nullptr, SB, g, Y, M, N, K, st);
    GemmParams p = {};
    p.Z = SB;
    p.fp4_g = g;
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    const int mt = M <= 64 ? 64 : 256;
    p.rows_per_tile = 128;
    p.n_row_tiles = ceil_div_i(N, 128);
    p.n_tok_tiles = ceil_div_i(M, mt);
    p.num_kb = ceil_div_i(K, 64);
    CUtensorMap tw, ts, tx;
    memset(&ts, 0, sizeof ts);
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)mt};
        if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        cuuint32_t box[2] = {8u, 128u};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_32B))
            return W4_ERR_CUDA;
    }
    const int64_t items = (int64_t)p.n_row_tiles * p.n_tok_tiles;
    if (items > (1 << 30)) return W4_ERR_UNSUPPORTED;
    if (mt == 64)
        return launch_cfg<64, 64, 8, 1, 8, 4, 2, false, false, false, false, false, FP4>(
            tw, ts, tx, p, (int)items, st);
    return launch_cfg<64, 256, 6, 1, 6, 2, 2, false, false, false, false, true, FP4>(
        tw, ts, tx, p, (int)items, st);
}

}  // namespace
}  // namespace w4

extern "C" w4_status w4a16_gemm_mxfp4(const w4_bf16 *X, const int32_t *Wq, const uint8_t *E,
                                      w4_bf16 *Y, int64_t M, int64_t N, int64_t K, void *stream) {
    return gemm_fp4<1>(X, Wq, E, 1.0f, Y, M, N, K, stream);
}

extern "C" w4_status w4a16_gemm_nvfp4(const w4_bf16 *X, const int32_t *Wq, const uint8_t *S,
                                      float g, w4_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                      void *stream) {
    return gemm_fp4<2>(X, Wq, S, g, Y, M, N, K, stream);
}

extern "C" int64_t w4_moe_capacity(int64_t T, int topk, int E, int block) {
    if (T < 0 || topk <= 0 || E <= 0 || block <= 0) return 0;
    const int64_t cap = T * topk + (int64_t)E * (block - 1);
    return (cap + block - 1) / block * block;
}

namespace w4 {
namespace {

// Grouped GEMM launch shared by the plain entry (silu_inter = 0: Y = C
// [num_slots, N]) and the SiLU*up entry (silu_inter = F, N = 2F: Y = H
// [num_slots, F]).
w4_status moe_launch(const w4_bf16 *A, int a_row_div, const int32_t *Wq, const w4_bf16 *S,
                     const int32_t *sorted_ids, const int32_t *expert_ids,
                     const int32_t *num_post_pad, int64_t cap, int block, int64_t num_slots,
                     w4_bf16 *Y, int64_t N, int64_t K, int E, int64_t silu_inter, void *stream,
                     int topk = 0, const float *comb_w = nullptr, w4_bf16 *comb_out = nullptr,
                     unsigned int *comb_cnt = nullptr) {
    if (!w4host::aligned16(A) || !w4host::aligned16(Wq) || !w4host::aligned16(S) ||
        !w4host::aligned16(sorted_ids) || !w4host::aligned16(expert_ids) ||
        !w4host::aligned16(num_post_pad) || !w4host::aligned16(Y))
        return W4_ERR_INVALID_ARG;
    if (a_row_div <= 0 || N <= 0 || K <= 0 || (K % 32) != 0 || E <= 0 || num_slots < 0 ||
        cap < 0 || block <= 0 || (cap % block) != 0)
        return W4_ERR_INVALID_ARG;
    if (block != 16 && block != 32 && block != 64) return W4_ERR_UNSUPPORTED;
    if ((K % 256) != 0) return W4_ERR_UNSUPPORTED;
    if (num_slots == 0 || cap == 0) return W4_OK;
    cudaStream_t st = (cudaStream_t)stream;

    GemmParams p = {};
    p.S = reinterpret_cast<const uint16_t *>(S);
    p.Y = reinterpret_cast<uint16_t *>(Y);
    p.A = reinterpret_cast<const uint16_t *>(A);
    p.sorted_ids = sorted_ids;
    p.expert_ids = expert_ids;
    p.num_post_pad = num_post_pad;
    p.M = num_slots;
    p.N = N;
    p.K = K;
    p.num_slots = num_slots;
    p.a_row_div = a_row_div;
    p.a_rows = (num_slots + a_row_div - 1) / a_row_div;
    if (cap / block > (1 << 30) || silu_inter > (1 << 28)) return W4_ERR_UNSUPPORTED;
    p.cap_blocks = (int)(cap / block);
    p.rows_per_tile = 128;
    p.silu_inter = (int)silu_inter;
    p.topk = topk;
    p.comb_w = comb_w;
    p.comb_out = reinterpret_cast<uint16_t *>(comb_out);
    p.comb_cnt = comb_cnt;
    // a SiLU*up tile covers 64 output columns (64 gate + 64 up rows)
    p.n_row_tiles = silu_inter > 0 ? ceil_div_i(silu_inter, 64) : ceil_div_i(N, 128);
    p.n_tok_tiles = 0;
    p.num_kb = ceil_div_i(K, 256);
    const cuuint32_t box_rows = silu_inter > 0 ? 64u : 128u;

    CUtensorMap tw, ts, tx;
    memset(&tx, 0, sizeof tx);
    {
        cuuint64_t dims[3] = {(cuuint64_t)(K / 8), (cuuint64_t)N, (cuuint64_t)E};
        cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N * (K / 2)};
        cuuint32_t box[3] = {32u, box_rows, 1u};
        if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return W4_ERR_CUDA;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)(K / 32), (cuuint64_t)N, (cuuint64_t)E};
        cuuint64_t strides[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N * (K / 16)};
        cuuint32_t box[3] = {8u, box_rows, 1u};
        if (!make_map(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, S, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return W4_ERR_CUDA;
    }
    // 32-slot blocks that the routing fills on average (>= 16 slots per expert)
    // run as they are.  Otherwise every block size runs on 16-slot work items:
    // an aligned block of 32 or 64 slots is block / 16 sub-blocks of the same
    // expert, and sub-blocks that hold only padding are skipped, so a wide
    // block costs what its real slots need (at decode sizes most of a wide
    // block is padding).
    if (block == 32 && num_slots >= 16 * E) {
        p.moe_mt = 32;
        p.moe_sub = 1;
        const int64_t items_max = (cap / 32) * p.n_row_tiles;
        const int items = (int)std::min<int64_t>(items_max, 1 << 30);
        return launch_cfg<256, 32, 6, 2, 2, 4, 2, true>(tw, ts, tx, p, items, st);
    }
    p.moe_mt = 16;
    p.moe_sub = block / 16;
    const int64_t items_max = (cap / 16) * p.n_row_tiles;
    const int items = (int)std::min<int64_t>(items_max, 1 << 30);
    return launch_cfg<256, 16, 6, 2, 3, 4, 2, true>(tw, ts, tx, p, items, st);
}

}  // namespace
}  // namespace w4

extern "C" w4_status w4_moe_w4a16_gemm(const w4_bf16 *A, int a_row_div, const int32_t *Wq,
                                       const w4_bf16 *S, const int32_t *sorted_ids,
                                       const int32_t *expert_ids, const int32_t *num_post_pad,
                                       int64_t cap, int block, int64_t num_slots, w4_bf16 *C,
                                       int64_t N, int64_t K, int E, void *stream) {
    return w4::moe_launch(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, cap, block,
                          num_slots, C, N, K, E, 0, stream);
}

extern "C" size_t w4_moe_combine_counter_bytes(int64_t T, int64_t N) {
    if (T <= 0 || N <= 0) return 0;
    return (size_t)T * (size_t)((N + 127) / 128) * 4 * sizeof(unsigned int);
}

extern "C" w4_status w4_moe_w4a16_gemm_combine(const w4_bf16 *A, const int32_t *Wq,
                                               const w4_bf16 *S, const int32_t *sorted_ids,
                                               const int32_t *expert_ids,
                                               const int32_t *num_post_pad, int64_t cap,
                                               int block, int topk, const float *w, w4_bf16 *C,
                                               unsigned int *counters, w4_bf16 *out, int64_t T,
                                               int64_t N, int64_t K, int E, void *stream) {
    if (topk < 1 || topk > 64 || T < 0 || w == nullptr || counters == nullptr ||
        (reinterpret_cast<uintptr_t>(counters) & 15u) != 0 || !w4host::aligned16(out))
        return W4_ERR_INVALID_ARG;
    if (T > ((int64_t)1 << 30) / topk) return W4_ERR_UNSUPPORTED;
    return w4::moe_launch(A, 1, Wq, S, sorted_ids, expert_ids, num_post_pad, cap, block,
                          T * topk, C, N, K, E, 0, stream, topk, w, out, counters);
}

extern "C" w4_status w4_moe_w4a16_gemm_silu(const w4_bf16 *A, int a_row_div, const int32_t *Wq,
                                            const w4_bf16 *S, const int32_t *sorted_ids,
                                            const int32_t *expert_ids,
                                            const int32_t *num_post_pad, int64_t cap, int block,
                                            int64_t num_slots, w4_bf16 *H, int64_t F, int64_t K,
                                            int E, void *stream) {
    if (F <= 0) return W4_ERR_INVALID_ARG;
    return w4::moe_launch(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, cap, block,
                          num_slots, H, 2 * F, K, E, F, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the decode GEMM.
//
// Some callers cannot give this library device memory for scratch: an
// inference engine that budgets every byte of device memory at start-up and
// forbids allocations afterwards, a plug-in whose host framework owns the
// allocator, or a caller that must not call cudaMalloc because it can
// synchronize the device.  w4a16_gemm_noalloc serves them with a fixed scratch
// array that lives in this library's device image: every GPU that loads the
// library holds these bytes until the process exits, and no call allocates.
// ---------------------------------------------------------------------------
namespace w4 {
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current (in host code the symbol is only a host-side stand-in).
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[64] = {nullptr};

w4_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        w4host::set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return W4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            w4host::set_cuda_error(e);
            return W4_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return W4_OK;
}

}  // namespace
}  // namespace w4

extern "C" w4_status w4a16_gemm_noalloc(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                                        w4_bf16 *Y, int64_t M, int64_t N, int64_t K, int group,
                                        void *stream) {
    if (group != 32) return W4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || (K % 32) != 0) return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    // Shapes the warp-level decode kernel takes need no scratch at all.
    if (w4host::gemv_supported(M, N, K))
        return w4a16_gemm(X, Wq, S, Y, M, N, K, group, nullptr, 0, stream);
    // The scratch this shape's schedule needs must fit the fixed array.
    SplitPlan sp;
    size_t need = 0, zero_bytes = 0;
    if (plan_split(M, N, K, w4host::num_sms(), &sp)) {
        need = sp.cnt_bytes + sp.part_bytes;
        zero_bytes = sp.cnt_bytes;
    }
    if (need > kNoAllocScratchBytes) return W4_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    const w4_status st = noalloc_scratch(&scratch);
    if (st != W4_OK) return st;
    // The split's arrival counters must start at zero; the array keeps whatever
    // the previous call (or an aborted one) left there.
    if (zero_bytes > 0) {
        const cudaError_t e = cudaMemsetAsync(scratch, 0, zero_bytes, (cudaStream_t)stream);
        if (e != cudaSuccess) {
            w4host::set_cuda_error(e);
            return W4_ERR_CUDA;
        }
    }
    return w4a16_gemm(X, Wq, S, Y, M, N, K, group, need > 0 ? scratch : nullptr,
                      need > 0 ? kNoAllocScratchBytes : 0, stream);
}
