// w4_moe_glue.cu -- the MoE layer around the grouped W4A16 GEMMs: router
// gating (softmax + top-k), the SiLU-gated product between the two GEMMs, and
// the weighted top-k combine after the second ([QAT] the fused gating kernel
// before moe_align_block_size and "MoE operator deep fusion"; [TAG] [35]).
// All three are HBM- or latency-bound elementwise/row kernels; each reads its
// inputs once with 16-byte (or per-row) accesses and writes its outputs once.
#include <cmath>

#include "w4_common.cuh"

namespace w4 {
namespace {

constexpr int kGateMaxE = 256;                 // 8 logits per lane
constexpr int kGateWarps = 8;                  // tokens per 256-thread block
constexpr int kGlueThreads = 256;

// One warp per token.  Ties in the order go to the lower expert id; the order
// is decided on the logits, which is the order of the exact probabilities.
__global__ void __launch_bounds__(32 * kGateWarps)
    gate_topk_kernel(const float *__restrict__ logits, int64_t T, int E, int topk,
                     int32_t *__restrict__ ids, float *__restrict__ weights) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kGateWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *l = logits + t * E;
    float v[kGateMaxE / 32];
#pragma unroll
    for (int i = 0; i < kGateMaxE / 32; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? __ldg(l + e) : -INFINITY;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kGateMaxE / 32; ++i) mx = fmaxf(mx, v[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kGateMaxE / 32; ++i)
        if (i * 32 + lane < E) sum += expf(v[i] - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    uint32_t taken = 0u;    // bit i: this lane's logit i * 32 + lane is selected
    for (int k = 0; k < topk; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < kGateMaxE / 32; ++i) {
            const int e = i * 32 + lane;
            if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            ids[t * topk + k] = bi;
            weights[t * topk + k] = expf(bv - mx) / sum;
        }
    }
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&b);
}

__device__ __forceinline__ float silu_times(float g, float u) {
    return (g / (1.0f + expf(-g))) * u;
}

// 8 outputs per thread: h[s, 8c .. 8c + 7] from gate_up[s, 8c ..] and
// gate_up[s, F + 8c ..].
__global__ void __launch_bounds__(kGlueThreads)
    silu_mul_kernel(const uint4 *__restrict__ gu, int64_t S, int64_t F8, uint4 *__restrict__ h) {
    const int64_t i = (int64_t)blockIdx.x * kGlueThreads + threadIdx.x;
    if (i >= S * F8) return;
    const int64_t s = i / F8, c = i - s * F8;
    const uint4 g = __ldg(gu + s * 2 * F8 + c);
    const uint4 u = __ldg(gu + s * 2 * F8 + F8 + c);
    uint4 o;
    o.x = pack_bf16x2(silu_times(bf16lo(g.x), bf16lo(u.x)), silu_times(bf16hi(g.x), bf16hi(u.x)));
    o.y = pack_bf16x2(silu_times(bf16lo(g.y), bf16lo(u.y)), silu_times(bf16hi(g.y), bf16hi(u.y)));
    o.z = pack_bf16x2(silu_times(bf16lo(g.z), bf16lo(u.z)), silu_times(bf16hi(g.z), bf16hi(u.z)));
    o.w = pack_bf16x2(silu_times(bf16lo(g.w), bf16lo(u.w)), silu_times(bf16hi(g.w), bf16hi(u.w)));
    h[i] = o;
}

// 8 outputs per thread: out[t, 8c .. 8c + 7] = sum_k w[t, k] * D[t*topk + k, ..],
// FP32, ascending k, products and sums each rounded once (no contraction).
__global__ void __launch_bounds__(kGlueThreads)
    combine_kernel(const uint4 *__restrict__ D, const float *__restrict__ w, int64_t T, int topk,
                   int64_t N8, uint4 *__restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * kGlueThreads + threadIdx.x;
    if (i >= T * N8) return;
    const int64_t t = i / N8, c = i - t * N8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < topk; ++k) {
        const float wk = __ldg(w + t * topk + k);
        const uint4 d = __ldg(D + (t * topk + k) * N8 + c);
        const uint32_t dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(wk, bf16lo(dv[q])));
            acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(wk, bf16hi(dv[q])));
        }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    out[i] = o;
}

int glue_grid(int64_t work) {
    return (int)std::max<int64_t>(1, std::min<int64_t>((work + kGlueThreads - 1) / kGlueThreads,
                                                        INT32_MAX));
}

}  // namespace
}  // namespace w4

extern "C" w4_status w4_moe_gate_topk(const float *logits, int64_t T, int E, int topk,
                                      int32_t *topk_ids, float *topk_weights, void *stream) {
    if (T < 0 || E < 1 || E > w4::kGateMaxE || topk < 1 || topk > E)
        return W4_ERR_INVALID_ARG;
    if (T == 0) return W4_OK;
    if (logits == nullptr || topk_ids == nullptr || topk_weights == nullptr)
        return W4_ERR_INVALID_ARG;
    if ((T + w4::kGateWarps - 1) / w4::kGateWarps > INT32_MAX) return W4_ERR_UNSUPPORTED;
    const int grid = (int)((T + w4::kGateWarps - 1) / w4::kGateWarps);
    w4::gate_topk_kernel<<<grid, 32 * w4::kGateWarps, 0, (cudaStream_t)stream>>>(
        logits, T, E, topk, topk_ids, topk_weights);
    return w4host::launch_status();
}

extern "C" int w4_moe_block_size(int64_t T, int topk, int E) {
    if (T <= 0 || topk <= 0 || E <= 0) return 0;
    const double load = (double)T * topk / E;
    return load <= 48.0 ? 16 : (load <= 96.0 ? 32 : 64);
}

extern "C" w4_status w4_silu_mul(const w4_bf16 *gate_up, int64_t S, int64_t F, w4_bf16 *h,
                                 void *stream) {
    if (S < 0 || F < 0 || (F % 8) != 0) return W4_ERR_INVALID_ARG;
    if (S == 0 || F == 0) return W4_OK;
    if (!w4host::aligned16(gate_up) || !w4host::aligned16(h)) return W4_ERR_INVALID_ARG;
    const int64_t work = S * (F / 8);
    w4::silu_mul_kernel<<<w4::glue_grid(work), w4::kGlueThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(gate_up), S, F / 8, reinterpret_cast<uint4 *>(h));
    return w4host::launch_status();
}

extern "C" w4_status w4_moe_combine(const w4_bf16 *D, const float *w, int64_t T, int topk,
                                    int64_t N, w4_bf16 *out, void *stream) {
    if (T < 0 || topk < 1 || N < 0 || (N % 8) != 0) return W4_ERR_INVALID_ARG;
    if (T == 0 || N == 0) return W4_OK;
    if (!w4host::aligned16(D) || !w4host::aligned16(out) || w == nullptr) return W4_ERR_INVALID_ARG;
    const int64_t work = T * (N / 8);
    w4::combine_kernel<<<w4::glue_grid(work), w4::kGlueThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(D), w, T, topk, N / 8, reinterpret_cast<uint4 *>(out));
    return w4host::launch_status();
}
