// w4_common.cuh -- shared device helpers of libw4a16 (sm_100a only).
//
// Thin inline-PTX wrappers for mbarriers, TMA tensor loads, cp.async and the
// 5th-generation tensor-core instructions (tcgen05.*), plus the bounded-wait
// and device-status machinery.  Every spin on an mbarrier is bounded by a
// global-timer deadline; on expiry the kernel records W4_ERR_TIMEOUT in the
// device status word and the calling role stops waiting.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/w4a16.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libw4a16 is built for sm_100a only"
#endif

namespace w4 {

// ---------------------------------------------------------------------------
// Device status word: set (never cleared) by kernels, read/cleared by the host
// through w4_device_status().  Each translation unit has its own copy (the
// library is built without relocatable device code); the one that kernels
// set is the GEMM's, read through w4host::gemm_device_status.
// ---------------------------------------------------------------------------
static __device__ unsigned int g_device_status = 0;

constexpr unsigned int kStatusTimeout = 1u;
// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_timeout() {
    atomicOr(&g_device_status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
        "r"(bytes)
        : "memory");
}

// try_wait with a suspend-time hint: a thread whose phase has not completed
// is suspended (it stops competing for issue slots) until the phase completes
// or the hint elapses, whichever comes first.
constexpr uint32_t kSuspendHintNs = 1000000u;   // 1 ms

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (after
// recording the timeout and raising *abort_flag) if the deadline passes or if
// another thread of the CTA already raised *abort_flag.
// The abort flag and the clock are looked at only every kPollsPerCheck polls:
// a poll is one mbarrier instruction, while the flag read and the clock read
// would add shared-memory and timer traffic that competes with the working
// warps' own shared-memory accesses.
constexpr uint32_t kPollsPerCheck = 64;
// Back-off between polls: a waiting warp then takes no issue slots and no
// shared-memory bandwidth from the warps doing the work, at the price of up to
// about this much extra latency when the phase completes.  Waiters off the
// critical path pass a longer back-off.
constexpr uint32_t kPollSleepNs = 32;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag,
                                          uint32_t sleep_ns = kPollSleepNs,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        __nanosleep(sleep_ns);
        if (n % kPollsPerCheck == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                record_timeout();
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Non-blocking test of the phase with the given parity (acquire on success).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait of a single thread on the critical path (the MMA issuer): a short spin
// of non-blocking tests, whose latency is well below that of a suspending
// try_wait when the phase is already complete, then the bounded wait above.
constexpr int kSpinTests = 64;
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity,
                                               volatile int *abort_flag) {
    for (int i = 0; i < kSpinTests; ++i)
        if (mbar_test(bar, parity)) return true;
    return mbar_wait(bar, parity, abort_flag);
}

// ---------------------------------------------------------------------------
// Proxy fences
// ---------------------------------------------------------------------------
// Generic-proxy shared-memory writes -> later async-proxy (TMA / tensor core) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A GEMM launched with programmatic stream
// serialization may become resident while the kernel before it on the stream
// still runs; it sets up its barriers and prefetches its tensor maps (kernel
// parameters), then waits here, before its first global-memory access, until
// that kernel has completed and its writes are visible.  Every such kernel
// reaches the wait on every path, so completion stays transitive along the
// stream.  The trigger lets the next kernel on the stream be scheduled as soon
// as every CTA of this one has started.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// L2 prefetch of a tensor-map box: a cache hint (no shared memory, no
// barrier, nothing returned), so it may run before the previous kernel on the
// stream completes; reads after griddep_wait() still see that kernel's writes.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *m, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// ---------------------------------------------------------------------------
// cp.async (16-byte global -> shared copies) with mbarrier completion
// ---------------------------------------------------------------------------
// Copies src_bytes (0 or 16) bytes and zero-fills the rest of the 16.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// The barrier receives one arrival once all prior cp.async of this thread land.
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// ---------------------------------------------------------------------------
// Tensor memory (tcgen05) -- cta_group::1 only
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warpgroup register resizing; all four warps of a warpgroup execute it.
// .inc waits until registers released by .dec elsewhere in the CTA cover it,
// so a split must fit in what the CTA was launched with.
template <int N>
__device__ __forceinline__ void reg_alloc() {
    static_assert(N % 8 == 0 && N >= 24 && N <= 256, "setmaxnreg range");
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
    static_assert(N % 8 == 0 && N >= 24 && N <= 256, "setmaxnreg range");
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
// From the launch count LAUNCH to N: .inc above it, .dec below it.
template <int N, int LAUNCH>
__device__ __forceinline__ void reg_set() {
    if constexpr (N > LAUNCH) reg_alloc<N>();
    else if constexpr (N < LAUNCH) reg_dealloc<N>();
}

// D[tmem] (+)= A[tmem] * B[smem desc]; kind::f16 (BF16 inputs, FP32 accumulator).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D (TMEM) (+)= A (shared memory, descriptor) * B (shared memory, descriptor).
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The barrier receives one arrival when all previously issued tcgen05.mma of
// this thread have completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// Store 8 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
}

// Store 16 / 32 consecutive 32-bit columns of this thread's TMEM lane (the wider
// forms move proportionally more bytes per instruction).
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
        "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Load 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// UMMA descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor for a K-major operand stored in the 128-byte
// swizzled canonical layout: rows of 128 bytes (64 BF16 along K), 8-row atoms
// of 1024 bytes stacked at a 1024-byte stride.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                           // leading byte offset (unused)
    d |= (uint64_t)(1024u >> 4) << 32;                 // stride byte offset: 8-row atom
    d |= (uint64_t)1u << 46;                           // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                           // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16, A = B = BF16, D = FP32, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t m, uint32_t n) {
    return (1u << 4)            // D format: F32
           | (1u << 7)          // A format: BF16
           | (1u << 10)         // B format: BF16
           | ((n >> 3) << 17)   // N / 8
           | ((m >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------------------
// INT4 -> BF16 unpack + dequant of one packed word (register level).
//
// Input: w = eight two's-complement codes q_0..q_7 (q_i in bits [4i, 4i+3]);
// s2 = the group's BF16 scale in both halves.  Output: four BF16x2 words,
// out[j] = (q_{2j} * s, q_{2j+1} * s), low half = even element.
//
// Step 1 (one LOP3 per pair): (w >> 4i) & 0x000F000F selects codes i and i+4;
// XOR with 0x43084308 flips the code's sign bit (two's complement -> offset
// binary, n ^ 8 = q + 8) and sets the BF16 exponent of 128, whose ulp is 1, so
// each half reads 136 + q exactly.  Step 2: byte permutes pair codes (2j,
// 2j+1).  Step 3: subtract 136 (exact), multiply by the scale (one rounding
// to nearest even: the product of a 4-bit and an 8-bit significand is exact
// before rounding), i.e. bf16_rne(q * s); q == 0 gives +0.0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    // (a & b) ^ c  -> truth table 0x6A
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t s2, uint32_t (&out)[4]) {
    const uint32_t m = 0x000F000Fu, x = 0x43084308u;
    uint32_t t0 = lop3_and_xor(w, m, x);          // codes 0, 4
    uint32_t t1 = lop3_and_xor(w >> 4, m, x);     // codes 1, 5
    uint32_t t2 = lop3_and_xor(w >> 8, m, x);     // codes 2, 6
    uint32_t t3 = lop3_and_xor(w >> 12, m, x);    // codes 3, 7
    uint32_t p01 = __byte_perm(t0, t1, 0x5410);
    uint32_t p23 = __byte_perm(t2, t3, 0x5410);
    uint32_t p45 = __byte_perm(t0, t1, 0x7632);
    uint32_t p67 = __byte_perm(t2, t3, 0x7632);
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
    const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
    uint32_t in[4] = {p01, p23, p45, p67};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&in[j]);
        v = __hsub2(v, bias);
        v = __hmul2(v, sc);
        out[j] = *reinterpret_cast<uint32_t *>(&v);
    }
}

// Unsigned codes with a zero point (asymmetric groups): OR-ing a nibble into
// BF16 128.0 (0x4300) gives 128 + q exactly; subtracting zb2 = (128 + z, 128 + z)
// leaves q - z exactly (|q - z| <= 15), and one multiply by the scale rounds
// (q - z) * s to BF16.  Same instruction count as dequant_word, natural order.
__device__ __forceinline__ void dequant_word_zp(uint32_t w, uint32_t s2, uint32_t zb2,
                                                uint32_t (&out)[4]) {
    const uint32_t m = 0x000F000Fu, x = 0x43004300u;
    uint32_t t0 = lop3_and_xor(w, m, x);          // codes 0, 4
    uint32_t t1 = lop3_and_xor(w >> 4, m, x);     // codes 1, 5
    uint32_t t2 = lop3_and_xor(w >> 8, m, x);     // codes 2, 6
    uint32_t t3 = lop3_and_xor(w >> 12, m, x);    // codes 3, 7
    uint32_t in[4] = {__byte_perm(t0, t1, 0x5410), __byte_perm(t2, t3, 0x5410),
                      __byte_perm(t0, t1, 0x7632), __byte_perm(t2, t3, 0x7632)};
    const __nv_bfloat162 zb = *reinterpret_cast<const __nv_bfloat162 *>(&zb2);
    const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&in[j]);
        v = __hsub2(v, zb);
        v = __hmul2(v, sc);
        out[j] = *reinterpret_cast<uint32_t *>(&v);
    }
}

// (128 + z) in both BF16 halves, z in [0, 15]: bits 0x4300 | z.
__device__ __forceinline__ uint32_t zp_bias2(uint32_t z) {
    const uint32_t h = 0x4300u | (z & 0xFu);
    return h | (h << 16);
}

// Same unpack without the pairing permutes: out[j] = (q_j * s, q_{j+4} * s).
// Used with activations whose 8-element chunks are stored in the matching order
// [x0, x4, x1, x5, x2, x6, x3, x7] (see permute_chunk8), which leaves the
// product unchanged because the K sum does not depend on the order of its terms.
__device__ __forceinline__ void dequant_word_k8perm(uint32_t w, uint32_t s2, uint32_t (&out)[4]) {
    const uint32_t m = 0x000F000Fu, x = 0x43084308u;
    uint32_t in[4];
    in[0] = lop3_and_xor(w, m, x);          // codes 0, 4
    in[1] = lop3_and_xor(w >> 4, m, x);     // codes 1, 5
    in[2] = lop3_and_xor(w >> 8, m, x);     // codes 2, 6
    in[3] = lop3_and_xor(w >> 12, m, x);    // codes 3, 7
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
    const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&in[j]);
        v = __hsub2(v, bias);
        v = __hmul2(v, sc);
        out[j] = *reinterpret_cast<uint32_t *>(&v);
    }
}

// dequant_word_k8perm for unsigned codes with a zero point (zb2 = zp_bias2(z)).
__device__ __forceinline__ void dequant_word_k8perm_zp(uint32_t w, uint32_t s2, uint32_t zb2,
                                                       uint32_t (&out)[4]) {
    const uint32_t m = 0x000F000Fu, x = 0x43004300u;
    uint32_t in[4];
    in[0] = lop3_and_xor(w, m, x);          // codes 0, 4
    in[1] = lop3_and_xor(w >> 4, m, x);     // codes 1, 5
    in[2] = lop3_and_xor(w >> 8, m, x);     // codes 2, 6
    in[3] = lop3_and_xor(w >> 12, m, x);    // codes 3, 7
    const __nv_bfloat162 zb = *reinterpret_cast<const __nv_bfloat162 *>(&zb2);
    const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&in[j]);
        v = __hsub2(v, zb);
        v = __hmul2(v, sc);
        out[j] = *reinterpret_cast<uint32_t *>(&v);
    }
}

// 8 BF16 values [x0..x7] (16 bytes) -> [x0, x4, x1, x5, x2, x6, x3, x7].
__device__ __forceinline__ uint4 permute_chunk8(uint4 v) {
    uint4 o;
    o.x = __byte_perm(v.x, v.z, 0x5410);
    o.y = __byte_perm(v.x, v.z, 0x7632);
    o.z = __byte_perm(v.y, v.w, 0x5410);
    o.w = __byte_perm(v.y, v.w, 0x7632);
    return o;
}

__device__ __forceinline__ uint32_t bf16x2_splat(uint16_t s) {
    return (uint32_t)s | ((uint32_t)s << 16);
}

// ---------------------------------------------------------------------------
// Micro-scaled FP4 (MR-GPTQ / QuTLASS FP4 summary: MXFP4 = 32 E2M1 values per
// power-of-two scale, NVFP4 = 16 per E4M3 scale under an FP32 tensor scale).
// Codes are packed like the INT4 codes: eight per int32, element i at bits
// [4i, 4i+3]; an E2M1 code is sign (bit 3), two exponent bits, one mantissa
// bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
// ---------------------------------------------------------------------------
// Two E2M1 codes (bits 0..3 and 4..7 of b) -> their values in FP32 (exact,
// through the hardware E2M1 -> FP16 conversion).
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t b, float &lo, float &hi) {
    uint32_t h;
    asm("{.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(b));
    float a, c;
    asm("{.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(a), "=f"(c)
        : "r"(h));
    lo = a;
    hi = c;
}

// An E4M3 byte (sign, 4 exponent bits with bias 7, 3 mantissa bits) -> FP32
// (exact, through the hardware E4M3 -> FP16 conversion).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t h;
    asm("{.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(b & 0xFFu));
    float a;
    asm("{.reg .f16 l, u;\n\tmov.b32 {l, u}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(a) : "r"(h));
    return a;
}

// 2^(E - 127) for a biased E8M0 exponent E in [0, 254] (E = 0: 2^-127, subnormal).
__device__ __forceinline__ float e8m0_to_f32(uint32_t E) {
    return __uint_as_float(E == 0u ? 0x00400000u : (E << 23));
}

__device__ __forceinline__ float fma_rn_f32(float a, float b, float c) {
    float d;
    asm("fma.rn.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// MXFP4: one packed word (8 codes) with the group's scale s = 2^(E - 127) ->
// four BF16x2 words of bf16_rne(value * s), natural order (out[j] = codes 2j,
// 2j + 1).  value * s is exact (a 2-bit significand times a power of two);
// the fused + 0 turns -0 into +0.
__device__ __forceinline__ void dequant_word_mxfp4(uint32_t w, float s, uint32_t (&out)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        e2m1x2_to_f32(w >> (8 * j), a, b);
        out[j] = f32x2_to_bf16x2(fma_rn_f32(a, s, 0.0f), fma_rn_f32(b, s, 0.0f));
    }
}

// NVFP4: one packed word with the group's E4M3 scale s8 (as FP32) and the
// tensor scale g -> bf16_rne(fl32(value * s8) * g): value * s8 is exact (2 and
// 4 significant bits), the product with g rounds once in FP32 (the added +0
// turns a product that underflows to -0 into +0), then BF16.
__device__ __forceinline__ void dequant_word_nvfp4(uint32_t w, float s8, float g,
                                                   uint32_t (&out)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        e2m1x2_to_f32(w >> (8 * j), a, b);
        out[j] = f32x2_to_bf16x2(__fadd_rn(__fmul_rn(fma_rn_f32(a, s8, 0.0f), g), 0.0f),
                                 __fadd_rn(__fmul_rn(fma_rn_f32(b, s8, 0.0f), g), 0.0f));
    }
}

}  // namespace w4

// ---------------------------------------------------------------------------
// Host-side helpers shared by the ABI entry points
// ---------------------------------------------------------------------------
namespace w4host {

void set_cuda_error(cudaError_t e);
// Reads the GEMM translation unit's device status word into *flag and clears it.
cudaError_t gemm_device_status(unsigned int *flag);
// Same for the warp-level MMA (decode) translation unit.
cudaError_t gemv_device_status(unsigned int *flag);

// Decode-shaped W4A16 GEMM on the warp-level MMA path (w4_gemv.cu): whether it
// takes the shape, and the launch (arguments already validated by the caller).
bool gemv_supported(int64_t M, int64_t N, int64_t K);
w4_status gemv_launch(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, w4_bf16 *Y,
                      int64_t M, int64_t N, int64_t K, void *stream);
// The same for zero-point groups (unsigned codes, Z one byte per group); also
// needs K % 512 == 0 (whole 16-byte lines of zero points per row) and a
// 16-byte-aligned Z, W4_ERR_UNSUPPORTED otherwise.
w4_status gemv_launch_zp(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z,
                         w4_bf16 *Y, int64_t M, int64_t N, int64_t K, void *stream);
// The same for FP4 codes (fp4 = 1: MXFP4 with E8M0 bytes, 2: NVFP4 with E4M3
// bytes under the tensor scale g); needs K % 512 == 0 and a 16-byte-aligned SB.
w4_status gemv_launch_fp4(int fp4, const w4_bf16 *X, const int32_t *Wq, const uint8_t *SB,
                          float g, w4_bf16 *Y, int64_t M, int64_t N, int64_t K, void *stream);

inline bool aligned16(const void *p) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline w4_status launch_status() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    return W4_OK;
}

int num_sms();

// Launch with programmatic stream serialization (the kernel must execute
// griddep_wait() before touching global memory; see w4::griddep_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
CUresult encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, cuuint32_t rank,
                      void *gaddr, const cuuint64_t *dims, const cuuint64_t *strides_bytes,
                      const cuuint32_t *box, CUtensorMapSwizzle swizzle);

}  // namespace w4host
