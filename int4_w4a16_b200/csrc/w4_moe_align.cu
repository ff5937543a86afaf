// w4_moe_align.cu -- moe_align_block_size on the GPU.
//
// INT4 QAT blog ("merge and align the tokens of the same expert";
// moe_align_block_size); reportify.cn "量化感知训练" [35].  Slot i = t*topk+k
// is routed to expert e_i.  Output: every expert's slots in ascending slot
// order, each run padded with the sentinel T*topk to a multiple of the block
// size, runs in ascending expert id; the expert of every block (-1 past the
// end); the padded total.
//
// One CTA of 32 warps, a stable counting sort without atomics (so the result
// is deterministic and unique):
//   1. warp w owns a contiguous chunk of the slots and counts its experts
//      32 slots at a time: __match_any_sync groups the lanes routed to the same
//      expert, and the group's lowest lane adds the group size to the warp's
//      private row of a shared [32, E] table;
//   2. one thread per expert turns its column into an exclusive prefix over the
//      warps (slots of expert e in earlier chunks) and the expert's total;
//   3. one warp scans the padded totals over the experts;
//   4. the outputs are pre-filled with the sentinel / -1, then every warp walks
//      its chunk again in slot order and writes each slot at
//      offset[e] + (slots of e in earlier chunks and earlier in this chunk),
//      i.e. in ascending slot order within each expert.
// Shared memory: 32 * E * 4 + 3 * E * 4 bytes; no global scratch.
#include <algorithm>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kAlignWarps = 32;
constexpr int kAlignThreads = kAlignWarps * 32;

__global__ void __launch_bounds__(kAlignThreads) moe_align_kernel(
    const int32_t *__restrict__ ids, int64_t n, int E, int block, int32_t *__restrict__ sorted_ids,
    int64_t cap, int32_t *__restrict__ expert_ids, int32_t *__restrict__ num_post_pad) {
    extern __shared__ uint32_t sm[];
    uint32_t *table = sm;                               // [32][E]: counts, then cursors
    uint32_t *offset = sm + (size_t)kAlignWarps * E;    // [E] padded exclusive offsets
    uint32_t *padded = offset + E;                      // [E]
    __shared__ uint32_t s_total_padded;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t chunk = ((n + kAlignWarps - 1) / kAlignWarps + 31) / 32 * 32;
    const int64_t lo = (int64_t)warp * chunk, hi = min(n, lo + chunk);
    uint32_t *row = table + (size_t)warp * E;

    for (int64_t i = tid; i < (int64_t)kAlignWarps * E; i += blockDim.x) table[i] = 0;
    __syncthreads();

    // 1. per-warp counts, 32 slots at a time (lanes past the chunk and
    //    out-of-range ids get a key of their own and are not counted)
    for (int64_t base = lo; base < hi; base += 32) {
        const int64_t i = base + lane;
        const int e = (i < hi) ? ids[i] : -1;
        const bool valid = e >= 0 && e < E;
        const int key = valid ? e : -1 - lane;
        const uint32_t grp = __match_any_sync(0xFFFFFFFFu, key);
        if (valid && lane == __ffs(grp) - 1) row[e] += __popc(grp);
        __syncwarp();
    }
    __syncthreads();

    // 2. per-expert exclusive prefix over the warps
    for (int e = tid; e < E; e += blockDim.x) {
        uint32_t run = 0;
        for (int w = 0; w < kAlignWarps; ++w) {
            const uint32_t c = table[(size_t)w * E + e];
            table[(size_t)w * E + e] = run;
            run += c;
        }
        padded[e] = (run + block - 1) / block * block;
    }
    __syncthreads();

    // 3. exclusive scan of the padded totals over the experts (warp 0)
    if (warp == 0) {
        const int per_lane = (E + 31) / 32;
        const int e0 = lane * per_lane, e1 = min(E, e0 + per_lane);
        uint32_t local = 0;
        for (int e = e0; e < e1; ++e) local += padded[e];
        uint32_t incl = local;
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += v;
        }
        uint32_t run = incl - local;
        for (int e = e0; e < e1; ++e) {
            offset[e] = run;
            run += padded[e];
        }
        if (lane == 31) s_total_padded = incl;
    }
    // 4a. sentinel / -1 pre-fill
    const int32_t sentinel = (int32_t)n;
    for (int64_t i = tid; i < cap; i += blockDim.x) sorted_ids[i] = sentinel;
    for (int64_t b = tid; b < cap / block; b += blockDim.x) expert_ids[b] = -1;
    __syncthreads();

    // 4b. stable scatter of the real slots
    for (int64_t base = lo; base < hi; base += 32) {
        const int64_t i = base + lane;
        const int e = (i < hi) ? ids[i] : -1;
        const bool valid = e >= 0 && e < E;
        const int key = valid ? e : -1 - lane;
        const uint32_t grp = __match_any_sync(0xFFFFFFFFu, key);
        uint32_t cursor = 0;
        if (valid) cursor = row[e];
        __syncwarp();
        if (valid) {
            sorted_ids[offset[e] + cursor + __popc(grp & lt_mask)] = (int32_t)i;
            if (lane == __ffs(grp) - 1) row[e] = cursor + __popc(grp);
        }
        __syncwarp();
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
    const int smem = (kAlignWarps * E + 2 * E) * 4;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(moe_align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (kAlignWarps + 2) * 1024 * 4) != cudaSuccess ||
            cudaFuncSetAttribute(moe_align_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return w4host::launch_status();
        configured = true;
    }
    moe_align_kernel<<<1, kAlignThreads, smem, (cudaStream_t)stream>>>(
        topk_ids, n, E, block, sorted_ids, cap, expert_ids, num_post_pad);
    return w4host::launch_status();
}
