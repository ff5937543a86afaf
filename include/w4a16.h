/*
 * w4a16.h -- C ABI of the B200 (sm_100a) library for group-wise INT4 weight
 * quantization and W4A16 inference (libw4a16.so).
 *
 * Sources, by page title and section:
 *   [QAT] SGLang RL team, "INT4 QAT end-to-end" blog (re-post): fake
 *         quantization with a straight-through estimator in Megatron
 *         (_FakeInt4QuantizationSTE), Fig. 4 "Rollout-side INT4 weight only"
 *         (eight INT4 values packed into one INT32: 8 x 4 bits = 32 bits,
 *         pack_int4_to_int32), "minimal packing and zero-overhead unpacking",
 *         moe_align_block_size, "MoE operator deep fusion".
 *   [TAG] reportify.cn concept page "量化感知训练": [8][9][16][17] fake
 *         quantization forward / STE backward, [10] real quantization of the
 *         exported weights, [11] 1x32 scale granularity, [32] W4A16 with two
 *         4-bit weights per byte, [35] moe_align_block_size.
 *   [BAS] "量化基础：从 FP32 到 INT4 的压缩艺术": §1.3 (INT4 range [-8, 7],
 *         BF16 1+8+7 bits), §2.2 (s = max|x| / q_max, q = clamp(round(x/s))),
 *         §2.4 (|x_hat - x| <= s/2), §6.2 (round half to even).
 *   [FP4] MR-GPTQ / QuTLASS FP4 summary page (NVFP4 / MXFP4 on Blackwell):
 *         MXFP4 = one shared power-of-two scale per 32 values (4.25 bits per
 *         value), NVFP4 = one FP8 scale per 16 values.
 *
 * Data formats (all row-major, all buffers owned by the caller):
 *   W    [rows, K]        BF16 weights (w4_bf16 = raw BF16 bits), K contiguous.
 *   S    [rows, K/32]     BF16 scales, one per group of 32 consecutive elements
 *                         along K: S = bf16_rne(fl32(amax / 7)).
 *   Wq   [rows, K/8]      int32 words; word j of a row holds codes
 *                         q[8j .. 8j+7], code i of the eight in bits
 *                         [4i, 4i+3] as a two's-complement nibble (low nibble
 *                         first).  q = clamp(rint_half_even(w / S), -8, 7).
 *   Wdq  [rows, K]        BF16 dequantized weights bf16_rne(q * S) (+0.0 for
 *                         q == 0).
 *   X    [M, K], Y [M, N] BF16 activations and outputs; Y = X . Wdq^T with
 *                         FP32 accumulation and one BF16 rounding.
 *
 * Conventions for every call:
 *   - Pointers are device pointers (cudaMalloc / PyTorch CUDA tensors) unless
 *     stated otherwise; they must be non-null and 16-byte aligned, or the call
 *     returns W4_ERR_INVALID_ARG without launching anything.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call validates its arguments on the host, then only
 *     enqueues kernels on `stream` and returns; it never synchronizes, never
 *     allocates device memory and keeps no pointer after it returns.  Scratch
 *     memory, where a schedule uses some, is passed in by the caller.
 *   - The GEMM kernels are launched with programmatic stream serialization:
 *     they may become resident while the previous kernel on `stream` still
 *     runs, but read and write no buffer (weights, scales, activations,
 *     outputs, workspace) before it has completed, so stream order is as for
 *     a plain launch.  Before that point they only set up shared memory and
 *     may issue L2 prefetches (cache hints) of their own weight tiles.
 *   - group must be 32 (else W4_ERR_UNSUPPORTED); K must be a positive
 *     multiple of 32.
 *   - A kernel launch failure returns W4_ERR_CUDA (w4_last_cuda_error() gives
 *     the cudaError_t).  Device-side waits are bounded: a kernel whose wait
 *     runs out sets a device status flag and exits cleanly; w4_device_status()
 *     reports it as W4_ERR_TIMEOUT.
 *   - Inputs are assumed finite; NaN / Inf inputs give unspecified codes.
 *   - Results are deterministic: run-to-run identical bits.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum w4_status {
    W4_OK = 0,
    W4_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or shape   */
    W4_ERR_UNSUPPORTED = 2, /* well-formed request outside what is built      */
    W4_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed            */
    W4_ERR_TIMEOUT = 4      /* a device-side bounded wait gave up             */
} w4_status;

typedef uint16_t w4_bf16; /* raw BF16 bits */

/* Library version (major * 10000 + minor * 100 + patch). */
int w4_version(void);

/* Human-readable name of a status code (static string). */
const char *w4_status_string(w4_status s);

/* The cudaError_t of the last W4_ERR_CUDA returned on this host thread. */
int w4_last_cuda_error(void);

/* Synchronizes `stream`, then reports and clears the device status flag:
 * W4_ERR_TIMEOUT if any kernel of this library gave up a bounded wait since
 * the last call, W4_ERR_CUDA if the synchronization itself failed, else W4_OK. */
w4_status w4_device_status(void *stream);

/* Self-test of the bounded device waits (an operational check of this
 * library; the pages have no counterpart).  Launches one warp on `stream`
 * that waits on a shared-memory mbarrier phase nothing completes, with the
 * same polling code as the GEMM's waits but a limit of `limit_us`
 * microseconds (1 .. 1e6).  The wait gives up, records the timeout and the
 * kernel exits, so the next w4_device_status() returns W4_ERR_TIMEOUT and the
 * CUDA context stays usable.  No memory is touched outside the kernel's own
 * shared memory.  Returns W4_ERR_INVALID_ARG for a limit out of range. */
w4_status w4_wait_selftest(uint32_t limit_us, void *stream);

/*
 * Fake quantization (QDQ) forward -- [QAT] fake quantization ("mapped to INT4
 * and immediately restored"), [TAG] [8][16], [BAS] §2.2.
 *   W    in   [rows, K] BF16
 *   Wdq  out  [rows, K] BF16, bf16_rne(q * S); may not alias W
 *   S    out  [rows, K/32] BF16 scales, or NULL to skip writing them
 * Memory-bound: reads 2 bytes and writes 2 (+1/16) bytes per element.
 */
w4_status w4_fake_quant(const w4_bf16 *W, w4_bf16 *Wdq, w4_bf16 *S,
                        int64_t rows, int64_t K, int group, void *stream);

/*
 * Straight-through-estimator backward -- [QAT] §2.1 (gradients skip the
 * rounding layer), [TAG] [9][17]: dW = dWdq bit for bit.  When dW == dWdq the
 * call is a no-op (zero-copy); otherwise it copies n BF16 values.
 */
w4_status w4_ste_backward(const w4_bf16 *dWdq, w4_bf16 *dW, int64_t n, void *stream);

/*
 * Real quantization + packing for export -- [TAG] [10][32], [QAT] Fig. 4.
 *   W    in   [rows, K] BF16
 *   Wq   out  [rows, K/8] int32, low-nibble-first two's-complement codes
 *   S    out  [rows, K/32] BF16 scales
 * The codes and scales are the same as w4_fake_quant's, so
 * w4_dequant(w4_quantize_pack(W)) == w4_fake_quant(W) bit for bit.
 */
w4_status w4_quantize_pack(const w4_bf16 *W, int32_t *Wq, w4_bf16 *S,
                           int64_t rows, int64_t K, int group, void *stream);

/*
 * Unpack + dequantize ([QAT] "zero-overhead unpacking"): Wdq = bf16_rne(q * S),
 * with the same register-level unpack the GEMMs use.  Mainly a test helper.
 */
w4_status w4_dequant(const int32_t *Wq, const w4_bf16 *S, w4_bf16 *Wdq,
                     int64_t rows, int64_t K, int group, void *stream);

/*
 * W4A16 GEMM -- [TAG] [32] (W4A16 inference), [QAT] Fig. 4 and "zero-overhead
 * unpacking"; the product runs on BF16 tensor cores with FP32 accumulation.
 *   X   in   [M, K] BF16        Wq  in  [N, K/8] int32   S  in  [N, K/32] BF16
 *   Y   out  [M, N] BF16, Y = X . dq(Wq, S)^T
 *   workspace, workspace_bytes: optional device scratch (256-byte aligned) for
 *        the decode-shaped split (M <= 64, K % 256 == 0, few 128-row tiles
 *        per SM).  NULL, or fewer bytes than w4a16_gemm_workspace_bytes(M, N, K)
 *        reports, selects the unsplit schedule instead (same results).  The
 *        workspace must be all zero before its first use; every call leaves
 *        its counters (the first 4 KB, whatever the shape) at zero again, so
 *        one workspace serves any sequence of shapes.  Calls that may overlap
 *        on the GPU must not share a workspace.  After W4_ERR_TIMEOUT, zero it
 *        again.
 * Any M >= 1, N >= 1.  Y may not alias an input.
 */
w4_status w4a16_gemm(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                     w4_bf16 *Y, int64_t M, int64_t N, int64_t K, int group,
                     void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace the split schedule of w4a16_gemm uses for this shape on
 * the current device (0 when that schedule does not apply).  Host-only. */
size_t w4a16_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * W4A16 GEMM for callers that cannot allocate device memory.  (The pages have
 * no counterpart: this is a deployment variant of w4a16_gemm.)
 *
 * Some callers cannot hand the library a workspace: an inference engine that
 * budgets all device memory at start-up and forbids later allocations, a
 * plug-in whose host framework owns the allocator, or code that must not call
 * cudaMalloc because it can synchronize the device.  This entry point computes
 * exactly what w4a16_gemm computes, using as its scratch a fixed 8 MiB array
 * inside the library's device image, which every GPU that loads the library
 * holds until the process exits.  It allocates nothing and calls no
 * allocating routine.
 *   - Shapes whose split schedule would need more than 8 MiB of scratch
 *     (e.g. M = 64 with K = 4096, N = 12288) return W4_ERR_UNSUPPORTED;
 *     w4a16_gemm with a caller-provided workspace handles them.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up per device); make that first call before any stream
 *     capture.
 *   - Every call shares the one array per device: the call zeroes the part that
 *     must start at zero (asynchronously, on `stream`), and calls that may
 *     overlap on the GPU (different streams) race on it and must be serialized
 *     by the caller.
 *   - The device address found at the first call is kept for the life of the
 *     process: it assumes the device's primary context is not reset
 *     (cudaDeviceReset) in between.
 *   - Shapes that w4a16_gemm runs without a split (1..8 rows with K a multiple
 *     of 256, or shapes too small to split) use no scratch and touch nothing.
 * Arguments as in w4a16_gemm.
 */
w4_status w4a16_gemm_noalloc(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S,
                             w4_bf16 *Y, int64_t M, int64_t N, int64_t K, int group,
                             void *stream);

/*
 * QAT forward GEMM with the fake quantization fused into the weight prologue
 * (the training-side counterpart of w4a16_gemm; INT4 QAT blog, fake
 * quantization in the forward pass; reportify.cn "量化感知训练" [8][16][62]):
 *     Y[m, n] = sum_k X[m, k] * Wdq[n, k],   Wdq = w4_fake_quant(W)  (group 32)
 * FP32 accumulation, one BF16 rounding, without ever writing Wdq: every
 * 128 x 64 tile of W is quantized and dequantized in registers (the exact
 * arithmetic of w4_fake_quant) on its way to the tensor cores.  The backward
 * pass of the straight-through estimator is dX = dY.Wdq (w4_qat_gemm_dx, below,
 * with the same fusion) and dW = dY^T.X (a plain BF16 GEMM that needs no
 * quantized weight, outside this library).
 *   X   in   [M, K] BF16;  W  in  [N, K] BF16 (the master weights);  Y  out  [M, N] BF16
 * K a multiple of 64 (W4_ERR_UNSUPPORTED otherwise; of 32: W4_ERR_INVALID_ARG);
 * group must be 32; 16-byte aligned, contiguous rows.
 */
w4_status w4_qat_gemm(const w4_bf16 *X, const w4_bf16 *W, w4_bf16 *Y, int64_t M, int64_t N,
                      int64_t K, int group, void *workspace, size_t workspace_bytes,
                      void *stream);

/*
 * QAT input gradient with the same fusion -- [QAT] fake quantization with a
 * straight-through estimator, [TAG] [8][9] (the backward pass through the fake-
 * quantized weight uses Wdq itself):
 *     dX[m, k] = sum_n dY[m, n] * Wdq[n, k],   Wdq = w4_fake_quant(W)  (group 32)
 * FP32 accumulation, one BF16 rounding, without writing Wdq: each 64 x 128
 * tile of W goes through the group QDQ in registers and is stored transposed
 * in shared memory as the A operand of tcgen05 BF16 MMAs (output rows = K).
 *   dY  in   [M, N] BF16;  W  in  [N, K] BF16 (the master weights);  dX  out  [M, K] BF16
 * K a multiple of 64 and N a multiple of 8 (W4_ERR_UNSUPPORTED otherwise; K
 * not a multiple of 32: W4_ERR_INVALID_ARG); group must be 32; 16-byte
 * aligned, contiguous rows.  N == 0 writes dX = 0.
 */
w4_status w4_qat_gemm_dx(const w4_bf16 *dY, const w4_bf16 *W, w4_bf16 *dX, int64_t M, int64_t N,
                         int64_t K, int group, void *workspace, size_t workspace_bytes,
                         void *stream);

/* Bytes of workspace the split schedule of the QAT GEMMs uses: up to 256 tokens
 * in one token tile and fewer 128-row output tiles than half the SMs (rows = N for
 * w4_qat_gemm, K for w4_qat_gemm_dx; contraction = K, resp. N) cut the
 * (row tile, 64-wide k-block) units evenly over the SMs and add the parked
 * FP32 partial sums in ascending k order (deterministic), as w4a16_gemm's
 * split does; 0 when the shape runs unsplit.  The workspace follows
 * w4a16_gemm's rules (256-byte aligned, all zero before its first use, left
 * with its counters zero; NULL or too small: unsplit, same results within
 * the GEMM tolerance).  Host-only. */
size_t w4_qat_gemm_workspace_bytes(int64_t M, int64_t rows, int64_t contraction);

/*
 * Asymmetric (zero-point) groups -- [BAS] §2.1 (affine map q = clamp(round(x/s)
 * + z, q_min, q_max), x^ = (q - z) * s) and §2.3 (s = (x_max - x_min) /
 * (q_max - q_min), z = clamp(round(q_min - x_min / s))), over the unsigned INT4
 * range q_min = 0, q_max = 15 of the GPTQ / AWQ formats (P1: "compatible with
 * GPTQ and AWQ").  Per group of 32 along K:
 *   s = bf16_rne(fl32(fl32(x_max - x_min) / 15)),
 *   z = clamp(rint_even(0 - fl32(x_min / s)), 0, 15),
 *   q = clamp(rint_even(fl32(x / s)) + z, 0, 15);  q = z = 0 when s == 0,
 *   x^ = bf16_rne((q - z) * s).
 *   W    in   [rows, K] BF16
 *   Wq   out  [rows, K/8] int32, low-nibble-first unsigned codes
 *   S    out  [rows, K/32] BF16 scales
 *   Z    out  [rows, K/32] uint8 zero points in [0, 15]
 * Same argument rules as w4_quantize_pack (Z: any alignment, not NULL).
 */
w4_status w4_quantize_pack_zp(const w4_bf16 *W, int32_t *Wq, w4_bf16 *S, uint8_t *Z,
                              int64_t rows, int64_t K, int group, void *stream);

/* Unpack + dequantize asymmetric groups: Wdq = bf16_rne((q - Z) * S). */
w4_status w4_dequant_zp(const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z, w4_bf16 *Wdq,
                        int64_t rows, int64_t K, int group, void *stream);

/*
 * W4A16 GEMM on asymmetric groups: Y[M, N] = X[M, K] . dequant_zp(Wq, S, Z)^T,
 * fp32 accumulation, BF16 output (the zero point is subtracted in the same
 * register unpack as w4a16_gemm's constant bias, no extra instruction).  1..8
 * rows with K % 512 == 0 and a 16-byte-aligned Z take the warp-level decode
 * kernel, 9..64 rows with K % 256 == 0 and a 16-byte-aligned Z the 256-wide
 * tensor-memory decode tiles (no workspace), every other shape the
 * tensor-memory kernel with 64-wide k-blocks.
 * K a multiple of 32; group 32; X, Wq, S, Y 16-byte aligned; Z not NULL.
 * Device pointers; the call is asynchronous on `stream`.
 */
w4_status w4a16_gemm_zp(const w4_bf16 *X, const int32_t *Wq, const w4_bf16 *S, const uint8_t *Z,
                        w4_bf16 *Y, int64_t M, int64_t N, int64_t K, int group, void *stream);

/*
 * ---------------------------------------------------------------------------
 * Micro-scaled FP4 weight groups -- [FP4] (MXFP4: groups of 32 with a power-of-
 * two scale; NVFP4: groups of 16 with an FP8 E4M3 scale); the activations stay
 * BF16, as in every W4A16 call.  The element is E2M1 (magnitudes 0, 0.5, 1,
 * 1.5, 2, 3, 4, 6; code = sign << 3 | magnitude index).  The page gives the
 * group sizes and scale types; the rest is read plainly:
 *   element code = nearest E2M1 value of w / step, ties to the even code,
 *                  saturating at 6, zero coded as +0;
 *   MXFP4 step   = 2^e, e = floor(log2 amax) - 2 clamped to [-127, 127],
 *                  stored as E = e + 127 (E8M0); all-zero group: E = 127;
 *   NVFP4 step   = e4m3(amax_group / (6 g)) * g, g = fl32(amax_tensor / 2688)
 *                  (1 for an all-zero tensor), E4M3 rounding nearest-even and
 *                  saturating at 448; a zero group scale stores zero codes;
 *   dequantized  = bf16_rne(fl32(fl32(value * s) * g))  (MXFP4: g = 1), +0.0
 *                  for a zero.
 *   Wq   [rows, K/8]  int32, eight 4-bit codes per word, low nibble first
 *   E    [rows, K/32] uint8 E8M0 exponents (MXFP4); 255 is not a valid scale
 *   S    [rows, K/16] uint8 E4M3 scales (NVFP4); 0x7F / 0xFF are not valid
 *   g    FP32 tensor scale (NVFP4)
 * K a positive multiple of 32; W, Wq, Wdq, X, Y 16-byte aligned; E, S any
 * alignment, not NULL.
 */
w4_status w4_quantize_pack_mxfp4(const w4_bf16 *W, int32_t *Wq, uint8_t *E, int64_t rows,
                                 int64_t K, void *stream);
w4_status w4_dequant_mxfp4(const int32_t *Wq, const uint8_t *E, w4_bf16 *Wdq, int64_t rows,
                           int64_t K, void *stream);
/* NVFP4 tensor scale of W[n] into *g (device float, 4-byte aligned):
 * g = fl32(max|W| / 2688), or 1 when W is all zero.  W 4-byte aligned. */
w4_status w4_nvfp4_tensor_scale(const w4_bf16 *W, int64_t n, float *g, void *stream);
/* NVFP4 codes and group scales of W under the tensor scale *g (device float,
 * as written by w4_nvfp4_tensor_scale). */
w4_status w4_quantize_pack_nvfp4(const w4_bf16 *W, const float *g, int32_t *Wq, uint8_t *S,
                                 int64_t rows, int64_t K, void *stream);
/* g is passed by value (host float). */
w4_status w4_dequant_nvfp4(const int32_t *Wq, const uint8_t *S, float g, w4_bf16 *Wdq,
                           int64_t rows, int64_t K, void *stream);
/*
 * W4A16 GEMM on FP4 weight groups: Y[M, N] = X[M, K] . Wdq^T with Wdq the
 * dequantized FP4 weights above, FP32 accumulation, one BF16 rounding.  The
 * codes are unpacked in registers (hardware E2M1 -> FP16 conversion, exact
 * FP32 scaling, BF16 rounding): 1..8 rows with K % 512 == 0 and 16-byte-
 * aligned scale bytes straight into warp-level MMA fragments (the decode
 * kernel of w4a16_gemm), other shapes into tensor memory as the A operand of
 * tcgen05 BF16 MMAs (9..64 rows with K % 256 == 0 on the 256-wide decode
 * tiles, the rest on the 64-wide tile), as in w4a16_gemm_zp.
 *   X in [M, K] BF16;  Wq in [N, K/8];  E in [N, K/32] / S in [N, K/16];
 *   Y out [M, N] BF16.  Device pointers; asynchronous on `stream`.
 */
w4_status w4a16_gemm_mxfp4(const w4_bf16 *X, const int32_t *Wq, const uint8_t *E, w4_bf16 *Y,
                           int64_t M, int64_t N, int64_t K, void *stream);
w4_status w4a16_gemm_nvfp4(const w4_bf16 *X, const int32_t *Wq, const uint8_t *S, float g,
                           w4_bf16 *Y, int64_t M, int64_t N, int64_t K, void *stream);

/* Padded capacity the caller must provide for w4_moe_align's sorted_ids:
 * T*topk + E*(block-1), rounded up to a multiple of block.  Host-only. */
int64_t w4_moe_capacity(int64_t T, int topk, int E, int block);

/*
 * moe_align_block_size -- [QAT] "merge and align the tokens routed to the same
 * expert", [TAG] [35].  Slot i = t*topk + k is routed to expert
 * topk_ids[t*topk + k].  Each expert's slots, in ascending slot order, form
 * one run padded up to a multiple of `block`; runs follow in ascending expert
 * id.
 *   topk_ids      in   [T, topk] int32 expert ids (ids outside [0, E) are skipped)
 *   sorted_ids    out  [cap] int32 slot ids; padding and the tail hold T*topk
 *   expert_ids    out  [cap/block] int32 expert of each block, -1 past the end
 *   num_post_pad  out  [1] int32 padded total (a multiple of block)
 * block must be a power of two in [1, 256]; cap >= w4_moe_capacity(...) and a
 * multiple of block; E in [1, 1024]; topk in [1, 64].  Single-block kernel
 * with no scratch memory.
 */
w4_status w4_moe_align(const int32_t *topk_ids, int64_t T, int topk, int E, int block,
                       int32_t *sorted_ids, int64_t cap, int32_t *expert_ids,
                       int32_t *num_post_pad, void *stream);

/*
 * Grouped W4A16 GEMM over the aligned slot list -- [QAT] "MoE operator deep
 * fusion", [TAG] [35].  For every block b < num_post_pad/block with expert
 * e = expert_ids[b], and every real slot = sorted_ids[b*block + j]
 * (slot < num_slots):
 *     C[slot, :] = A[slot / a_row_div, :] . dq(Wq[e], S[e])^T
 *   A             in   [ceil(num_slots / a_row_div), K] BF16 (tokens for the
 *                      gate_up projection with a_row_div = topk; per-slot
 *                      rows for the down projection with a_row_div = 1)
 *   Wq, S         in   [E, N, K/8] int32, [E, N, K/32] BF16
 *   sorted_ids, expert_ids, num_post_pad   in (device), as written by w4_moe_align
 *   C             out  [num_slots, N] BF16; rows of padding slots are never written
 * block must be one of 16, 32, 64; cap is the length of sorted_ids.  The
 * number of blocks is read on the device, so the call needs no host sync.
 */
w4_status w4_moe_w4a16_gemm(const w4_bf16 *A, int a_row_div, const int32_t *Wq,
                            const w4_bf16 *S, const int32_t *sorted_ids,
                            const int32_t *expert_ids, const int32_t *num_post_pad,
                            int64_t cap, int block, int64_t num_slots, w4_bf16 *C,
                            int64_t N, int64_t K, int E, void *stream);

/*
 * Grouped W4A16 GEMM for the gate_up projection with the SiLU-gated product
 * fused into its epilogue ([QAT] "MoE operator deep fusion"): for every real
 * slot of every aligned block (as in w4_moe_w4a16_gemm), with the slot's FP32
 * sums g = A.dq(W_e)[j]^T and u = A.dq(W_e)[F + j]^T,
 *     H[slot, j] = bf16( silu(g) * u ),  silu(x) = x / (1 + exp(-x))   (FP32)
 * i.e. w4_silu_mul applied to the unrounded gate_up sums, without writing them.
 *   Wq, S   in   [E, 2F, K/8] int32, [E, 2F, K/32] BF16: rows 0..F-1 gate, F..2F-1 up
 *   H       out  [num_slots, F] BF16; rows of padding slots are never written
 * Other arguments and constraints as in w4_moe_w4a16_gemm.
 */
w4_status w4_moe_w4a16_gemm_silu(const w4_bf16 *A, int a_row_div, const int32_t *Wq,
                                 const w4_bf16 *S, const int32_t *sorted_ids,
                                 const int32_t *expert_ids, const int32_t *num_post_pad,
                                 int64_t cap, int block, int64_t num_slots, w4_bf16 *H,
                                 int64_t F, int64_t K, int E, void *stream);

/*
 * ---------------------------------------------------------------------------
 * MoE layer around the grouped GEMMs.  The pages name the pieces without
 * defining them: a fused gating kernel (softmax + top-k), a block size chosen
 * from the token count and the expert histogram, and the fusion of the MoE
 * operators ([QAT] "moe_align_block_size", "MoE operator deep fusion"; [TAG]
 * [35]).  The readings below are the plainest ones the pages allow.
 * ---------------------------------------------------------------------------
 */

/*
 * Router gating: softmax over the E logits of each token, then the topk
 * experts with the largest probability, in descending order, ties to the
 * lower expert id.  The order is decided on the logits (softmax is strictly
 * increasing in the logit, so this is the order of the exact probabilities;
 * no rounding of an exponential decides an id).  The weights are the selected
 * probabilities, not renormalized over the topk:
 *     p[t, e] = exp(l[t, e] - max_e l[t, e]) / sum_e exp(l[t, e] - max_e l[t, e])   (FP32)
 *   logits        in   [T, E] FP32 (finite)
 *   topk_ids      out  [T, topk] int32
 *   topk_weights  out  [T, topk] FP32
 * E in [1, 256], topk in [1, E].  One warp per token.
 */
w4_status w4_moe_gate_topk(const float *logits, int64_t T, int E, int topk, int32_t *topk_ids,
                           float *topk_weights, void *stream);

/*
 * Block size for w4_moe_align / w4_moe_w4a16_gemm from the routing's average
 * load per expert (T * topk / E): 16 up to 48 slots per expert, 32 up to 96,
 * 64 beyond.  The grouped GEMM runs blocks of 32 and 64 as 16-slot sub-blocks
 * and skips the padding ones, so small blocks cost least at decode sizes
 * (measured on B200 at T = 16, 64, 256 with 128 experts, top-8: block 16 was
 * fastest or within 5 %); wider blocks only pay off when they are filled.
 * Host-only; returns 0 for invalid arguments.
 */
int w4_moe_block_size(int64_t T, int topk, int E);

/*
 * SiLU-gated product between the two grouped GEMMs: for each row s,
 *     h[s, j] = bf16( silu(g) * u ),  g = gate_up[s, j], u = gate_up[s, F + j],
 *     silu(x) = x / (1 + exp(-x))   (FP32)
 *   gate_up   in   [S, 2F] BF16 (the gate rows of the expert weights first)
 *   h         out  [S, F] BF16
 * F a multiple of 8; rows are 16-byte aligned.
 */
w4_status w4_silu_mul(const w4_bf16 *gate_up, int64_t S, int64_t F, w4_bf16 *h, void *stream);

/*
 * Weighted top-k combine after the down projection:
 *     out[t, n] = bf16( sum_{k = 0..topk-1} w[t, k] * D[t * topk + k, n] )
 * accumulated in FP32 in ascending k, each product rounded before its add.
 *   D       in   [T * topk, N] BF16 (slot rows, slot = t * topk + k)
 *   w       in   [T, topk] FP32
 *   out     out  [T, N] BF16
 * N a multiple of 8.
 */
w4_status w4_moe_combine(const w4_bf16 *D, const float *w, int64_t T, int topk, int64_t N,
                         w4_bf16 *out, void *stream);

/*
 * Down projection with the weighted top-k combine fused into its epilogue
 * ([QAT] "MoE operator deep fusion"): w4_moe_w4a16_gemm with a_row_div = 1 and
 * num_slots = T * topk, writing C as that call does, and in the same kernel
 *     out[t, n] = bf16( sum_{k ascending} w[t, k] * C[t * topk + k, n] )
 * with w4_moe_combine's arithmetic (every product and sum rounded once, FP32),
 * so out is bit for bit what w4_moe_combine gives on this C.  The last work
 * item to finish a token's rows does the sum: an arrival counter per (token,
 * 128-row tile, 32-row quarter) in `counters` decides which, so the result does
 * not depend on the order in which work items finish.
 *   w         in   [T, topk] FP32 routing weights (device)
 *   counters  in/out  w4_moe_combine_counter_bytes(T, N) bytes (device, 16-byte
 *                  aligned), all zero before the first call; every call leaves
 *                  them zero again (zero them again after W4_ERR_TIMEOUT)
 *   out       out  [T, N] BF16
 * Every slot must be routed to an expert in [0, E) (w4_moe_gate_topk's ids
 * are): a token with a skipped slot never completes and its out row is not
 * written.  Other arguments and constraints as in w4_moe_w4a16_gemm; topk in
 * [1, 64].
 */
size_t w4_moe_combine_counter_bytes(int64_t T, int64_t N);
w4_status w4_moe_w4a16_gemm_combine(const w4_bf16 *A, const int32_t *Wq, const w4_bf16 *S,
                                    const int32_t *sorted_ids, const int32_t *expert_ids,
                                    const int32_t *num_post_pad, int64_t cap, int block,
                                    int topk, const float *w, w4_bf16 *C, unsigned int *counters,
                                    w4_bf16 *out, int64_t T, int64_t N, int64_t K, int E,
                                    void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
