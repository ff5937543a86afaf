"""Parity of the asymmetric (zero-point) group path with the CPU oracle: the
quantizer and dequant bit for bit, the W4A16 GEMM on zero-point groups within
the GEMM tolerance and bit for bit on one-hot activations (quantization
tutorial §2.1 affine map, §2.3 asymmetric scale and zero point)."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits
from tests.test_gpu_parity import DEV, assert_gemm_close

pytestmark = pytest.mark.gpu


def _edge_weights(N, K, seed):
    """Ordinary groups next to each special case of the asymmetric map."""
    W = synth.normal_bf16((N, K), 0.02, seed=seed, outlier_frac=0.01).clone()
    if N > 8 and K >= 256:
        W[0, 0:32] = 0.0                                                # s = 0
        W[1, 32:64] = 0.75                                              # constant: s = 0
        W[2, 64:96] = torch.linspace(1.0, 2.0, 32).to(torch.bfloat16)   # all positive: z -> 0
        W[3, 96:128] = torch.linspace(-2.0, -1.0, 32).to(torch.bfloat16)  # all negative: z -> 15
        W[4, 128:160] = torch.tensor([float(i % 16 - 5) for i in range(32)]).to(torch.bfloat16)
        W[5, 160:192] = torch.linspace(100.0, 100.5, 32).to(torch.bfloat16)  # narrow, far from 0
        W[6, 192:224] = 1e-39 * torch.linspace(-1, 1, 32).to(torch.bfloat16)  # subnormal range
        W[7, 224:256] = torch.tensor([0.25 * (i % 7 - 3) for i in range(32)]).to(torch.bfloat16)
    if N > 13:
        t = 2.0 ** -126
        groups = {
            # s = 1, z = 7: exact ties x / s = k + 1/2 of both parities
            8: [-7.0, 8.0] + [k + 0.5 for k in range(-7, 8)] + [float(k) for k in range(-6, 8)] + [0.0],
            # s = 0.5, z = 7: ties at odd multiples of 0.25
            9: [-3.5, 4.0] + [0.25 * (2 * k + 1) for k in range(-7, 8)] + [0.5 * k for k in range(-6, 8)] + [0.0],
            # s = 1.5 (significand 192): ties at odd multiples of 0.75
            10: [-10.5, 12.0] + [0.75 * (2 * k + 1) for k in range(-7, 8)] + [1.5 * k for k in range(-6, 8)] + [0.0],
            # all negative: z = 15, ties below zero
            11: [-15.0, 0.0] + [-(k + 0.5) for k in range(15)] + [-float(k) for k in range(1, 15)] + [-7.0],
            # s = 2^-126, the smallest scale of the reciprocal path: ties of subnormal weights
            12: [0.0, 15 * t] + [(k + 0.5) * t for k in range(15)] + [k * t for k in range(1, 15)] + [7 * t],
            # s = 2^101, above the reciprocal path's range: IEEE divisions
            13: [-7 * 2.0 ** 101, 8 * 2.0 ** 101] + [(k + 0.5) * 2.0 ** 101 for k in range(-7, 8)]
                + [k * 2.0 ** 101 for k in range(-6, 8)] + [0.0],
        }
        for row, vals in groups.items():
            assert len(vals) == 32
            W[row, 0:32] = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    return W


@pytest.mark.parametrize("rows,K", [(1, 32), (9, 256), (300, 640), (1000, 4096), (4097, 256)])
def test_quantize_pack_zp_bit_exact(rows, K):
    W = _edge_weights(rows, K, seed=rows + K)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    w4.w4_device_status()
    oWq, oS, oZ = oracle.quantize_pack_zp(bits(W))
    assert np.array_equal(Wq.cpu().numpy(), oWq)
    assert np.array_equal(bits(S), oS)
    assert np.array_equal(Z.cpu().numpy(), oZ)
    Wdq = bits(w4.dequant_zp(Wq, S, Z))
    assert np.array_equal(Wdq, oracle.dequant_zp(oWq, oS, oZ))


def test_quantize_pack_zp_layer_shape():
    """The prefill layer's weights (18432 x 7168): every output compared."""
    W = synth.normal_bf16((18432, 7168), 0.02, seed=3, outlier_frac=0.001)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    oWq, oS, oZ = oracle.quantize_pack_zp(bits(W))
    assert np.array_equal(Wq.cpu().numpy(), oWq)
    assert np.array_equal(bits(S), oS)
    assert np.array_equal(Z.cpu().numpy(), oZ)


# 9..64 rows with K % 256 == 0 take the 256-wide decode tiles (zero points read
# directly by the dequant warps): 16-, 32- and 64-token tiles, ragged N and M,
# more row tiles than SMs
@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (1, 300, 4096), (5, 100, 128), (64, 300, 640),
                                   (65, 257, 256), (300, 1000, 1024), (512, 1024, 2048),
                                   (3, 129, 96), (16, 300, 4096), (9, 1000, 1024),
                                   (32, 4099, 2048), (64, 129, 768), (24, 12288, 4096),
                                   (17, 20000, 512)])
def test_gemm_zp_shapes(M, N, K):
    W = _edge_weights(N, K, seed=M + N + K)
    X = synth.normal_bf16((M, K), 1.0, seed=M + 7)
    oWq, oS, oZ = oracle.quantize_pack_zp(bits(W))
    Y = bits(w4.gemm_zp(X.to(DEV), torch.from_numpy(oWq).to(DEV),
                        torch.from_numpy(oS.view(np.int16)).view(torch.bfloat16).to(DEV),
                        torch.from_numpy(oZ).to(DEV)))
    w4.w4_device_status()
    _, R = oracle.w4a16_gemm_zp(bits(X), oWq, oS, oZ)
    assert_gemm_close(Y, R, f"zp M={M} N={N} K={K}")


def test_gemm_zp_one_hot_exact():
    """X = identity rows: Y[m, n] = dequant_zp(W)[n, m] bit for bit."""
    N, K = 200, 256
    W = _edge_weights(N, K, seed=21)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    Wdq = oracle.dequant_zp(Wq.cpu().numpy(), bits(S), Z.cpu().numpy())
    for m0 in range(0, K, 64):
        X = torch.zeros((64, K), dtype=torch.bfloat16)
        X[torch.arange(64), m0 + torch.arange(64)] = 1.0
        Y = bits(w4.gemm_zp(X.to(DEV), Wq, S, Z))
        want = Wdq[:, m0:m0 + 64].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch at m0={m0}: {bad[:8].tolist()}")
    w4.w4_device_status()


def test_gemm_zp_layer_sampled():
    """The prefill layer's weights (N = 18432, K = 7168) at M = 16; every 97th
    output row against the oracle's GEMM on the same codes."""
    N, K, M = 18432, 7168, 16
    W = synth.normal_bf16((N, K), 0.02, seed=5, outlier_frac=0.001)
    X = synth.normal_bf16((M, K), 1.0, seed=6)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    Y = bits(w4.gemm_zp(X.to(DEV), Wq, S, Z))
    rows = np.arange(0, N, 97)
    _, R = oracle.w4a16_gemm_zp(bits(X), Wq.cpu().numpy()[rows], bits(S)[rows],
                                Z.cpu().numpy()[rows])
    assert_gemm_close(Y[:, rows], R, "zp layer")


@pytest.mark.parametrize("M,N,K", [(1, 333, 512), (3, 257, 1024), (8, 1000, 4096),
                                   (5, 64, 4608), (8, 129, 2560), (2, 12288, 4096)])
def test_gemm_zp_decode_kernel(M, N, K):
    """1..8 rows with K % 512 == 0 take the warp-level MMA kernel (zero points by
    TMA beside the scales); one to three passes over K, ragged N."""
    W = _edge_weights(N, K, seed=M * 7 + N + K)
    X = synth.normal_bf16((M, K), 1.0, seed=M + 11)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    Y = bits(w4.gemm_zp(X.to(DEV), Wq, S, Z))
    w4.w4_device_status()
    _, R = oracle.w4a16_gemm_zp(bits(X), Wq.cpu().numpy(), bits(S), Z.cpu().numpy())
    assert_gemm_close(Y, R, f"zp decode M={M} N={N} K={K}")


def test_gemm_zp_decode_kernel_one_hot_exact():
    """X = 8 identity rows through the warp-level kernel: Y[m, n] =
    dequant_zp(W)[n, m] bit for bit."""
    N, K = 300, 1024
    W = _edge_weights(N, K, seed=33)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    Wdq = oracle.dequant_zp(Wq.cpu().numpy(), bits(S), Z.cpu().numpy())
    for m0 in range(0, K, 8 * 16):
        X = torch.zeros((8, K), dtype=torch.bfloat16)
        X[torch.arange(8), m0 + torch.arange(8)] = 1.0
        Y = bits(w4.gemm_zp(X.to(DEV), Wq, S, Z))
        want = Wdq[:, m0:m0 + 8].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch at m0={m0}: {bad[:8].tolist()}")
    w4.w4_device_status()


def test_gemm_zp_unaligned_zero_points_take_the_tensor_memory_kernel():
    """Zero points not 16-byte aligned: the decode kernel declines, the
    tensor-memory kernel computes the same product."""
    N, K, M = 200, 1024, 4
    W = _edge_weights(N, K, seed=44)
    X = synth.normal_bf16((M, K), 1.0, seed=45)
    Wq, S, Z = w4.quantize_pack_zp(W.to(DEV))
    Zbuf = torch.empty(Z.numel() + 16, dtype=torch.uint8, device=DEV)
    Zoff = Zbuf[1:1 + Z.numel()].view(Z.shape)
    Zoff.copy_(Z)
    Y = bits(w4.gemm_zp(X.to(DEV), Wq, S, Zoff))
    w4.w4_device_status()
    _, R = oracle.w4a16_gemm_zp(bits(X), Wq.cpu().numpy(), bits(S), Z.cpu().numpy())
    assert_gemm_close(Y, R, "zp unaligned Z")
