// w4_moe_align.cu -- moe_align_block_size on the GPU.
//
// INT4 QAT blog ("merge and align the tokens of the same expert";
// moe_align_block_size); reportify.cn "量化感知训练" [35].  Slot i = t*topk+k
// is routed to expert e_i.  Output: every expert's slots in ascending slot
// order, each run padded with the sentinel T*topk to a multiple of the block
// size, runs in ascending expert id; the expert of every block (-1 past the
// end); the padded total.
//
// One CTA, a stable counting sort without atomics (so the result is
// deterministic and unique):
//   1. the slots are cut into NR contiguous ranges, one per "range thread";
//      each range thread counts its experts into a private row of a shared
//      [NR, E] table;
//   2. one thread per expert turns its column into an exclusive prefix over
//      the ranges (slots of expert e in earlier ranges) and the total;
//   3. the padded totals are scanned over the experts (one warp);
//   4. the outputs are pre-filled with the sentinel / -1, then every range
//      thread walks its range in order and writes slot ids at
//      offset[e] + (slots of e before it) -- ascending slot order within each
//      expert, because ranges are contiguous and walked in order.
// Shared memory: NR * E * 4 bytes + 3 * E * 4 bytes; no global scratch.
#include <algorithm>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kAlignThreads = 1024;
constexpr int kTableBytes = 160 * 1024;

__global__ void __launch_bounds__(kAlignThreads) moe_align_kernel(
    const int32_t *__restrict__ ids, int64_t n, int E, int block, int NR, int32_t *__restrict__ sorted_ids,
    int64_t cap, int32_t *__restrict__ expert_ids, int32_t *__restrict__ num_post_pad) {
    extern __shared__ uint32_t sm[];
    uint32_t *table = sm;                           // [NR][E]
    uint32_t *total = sm + (size_t)NR * E;          // [E]
    uint32_t *offset = total + E;                   // [E] padded exclusive offsets
    uint32_t *padded = offset + E;                  // [E]
    __shared__ uint32_t s_total_padded;

    const int tid = threadIdx.x;
    const int64_t per = (n + NR - 1) / NR;

    for (int64_t i = tid; i < (int64_t)NR * E; i += blockDim.x) table[i] = 0;
    __syncthreads();

    // 1. private per-range counts
    if (tid < NR) {
        const int64_t lo = (int64_t)tid * per, hi = min(n, lo + per);
        uint32_t *row = table + (size_t)tid * E;
        for (int64_t i = lo; i < hi; ++i) {
            const int e = ids[i];
            if (e >= 0 && e < E) row[e] += 1;
        }
    }
    __syncthreads();

    // 2. per-expert exclusive prefix over the ranges
    for (int e = tid; e < E; e += blockDim.x) {
        uint32_t run = 0;
        for (int r = 0; r < NR; ++r) {
            const uint32_t c = table[(size_t)r * E + e];
            table[(size_t)r * E + e] = run;
            run += c;
        }
        total[e] = run;
        padded[e] = (run + block - 1) / block * block;
    }
    __syncthreads();

    // 3. exclusive scan of the padded totals over the experts (warp 0)
    if (tid < 32) {
        const int per_lane = (E + 31) / 32;
        const int e0 = tid * per_lane, e1 = min(E, e0 + per_lane);
        uint32_t local = 0;
        for (int e = e0; e < e1; ++e) local += padded[e];
        uint32_t incl = local;
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (tid >= d) incl += v;
        }
        uint32_t run = incl - local;
        for (int e = e0; e < e1; ++e) {
            offset[e] = run;
            run += padded[e];
        }
        if (tid == 31) s_total_padded = incl;
    }
    // 4a. sentinel / -1 pre-fill
    const int32_t sentinel = (int32_t)n;
    for (int64_t i = tid; i < cap; i += blockDim.x) sorted_ids[i] = sentinel;
    for (int64_t b = tid; b < cap / block; b += blockDim.x) expert_ids[b] = -1;
    __syncthreads();

    // 4b. stable scatter of the real slots
    if (tid < NR) {
        const int64_t lo = (int64_t)tid * per, hi = min(n, lo + per);
        uint32_t *row = table + (size_t)tid * E;
        for (int64_t i = lo; i < hi; ++i) {
            const int e = ids[i];
            if (e >= 0 && e < E) {
                const uint32_t pos = offset[e] + row[e];
                row[e] += 1;
                sorted_ids[pos] = (int32_t)i;
            }
        }
    }
    // 4c. block -> expert
    for (int e = tid; e < E; e += blockDim.x) {
        const uint32_t b0 = offset[e] / block, b1 = (offset[e] + padded[e]) / block;
        for (uint32_t b = b0; b < b1; ++b) expert_ids[b] = e;
    }
    if (tid == 0) *num_post_pad = (int32_t)s_total_padded;
}

}  // namespace
}  // namespace w4

using namespace w4;

extern "C" w4_status w4_moe_align(const int32_t *topk_ids, int64_t T, int topk, int E, int block,
                                  int32_t *sorted_ids, int64_t cap, int32_t *expert_ids,
                                  int32_t *num_post_pad, void *stream) {
    if (T < 0 || topk <= 0 || topk > 64 || E <= 0 || E > 1024 || block <= 0 || block > 256 ||
        (block & (block - 1)) != 0)
        return W4_ERR_INVALID_ARG;
    if (T * topk > (int64_t)INT32_MAX / 2) return W4_ERR_UNSUPPORTED;
    if (cap < w4_moe_capacity(T, topk, E, block) || (cap % block) != 0) return W4_ERR_INVALID_ARG;
    if ((T > 0 && !w4host::aligned16(topk_ids)) || !w4host::aligned16(sorted_ids) ||
        !w4host::aligned16(expert_ids) || !w4host::aligned16(num_post_pad))
        return W4_ERR_INVALID_ARG;
    const int64_t n = T * topk;
    int NR = std::min<int64_t>(kAlignThreads, kTableBytes / (4 * (int64_t)E));
    NR = std::max(1, std::min<int>(NR, (int)std::max<int64_t>(1, n)));
    const int smem = (NR * E + 3 * E) * 4;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(moe_align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kTableBytes + 3 * 4 * 1024 + 1024) != cudaSuccess)
            return w4host::launch_status();
        configured = true;
    }
    moe_align_kernel<<<1, kAlignThreads, smem, (cudaStream_t)stream>>>(
        topk_ids, n, E, block, NR, sorted_ids, cap, expert_ids, num_post_pad);
    return w4host::launch_status();
}
