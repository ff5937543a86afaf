"""Parity of the decode-shaped W4A16 GEMM with the CPU oracle, through the C
ABI.  1..8 activation rows with K a multiple of 256 take the warp-level MMA
kernel (w4_gemv.cu); the other shapes here run the tensor-memory kernel at
the same sizes (its stream-K split included, on one shared workspace).

Shapes cover every launch configuration of the warp-level kernel: one and
several passes of the warps over K (4096 each), with a partly idle last pass;
row ranges of one to six 16-row tiles per CTA,
including ones whose stages outnumber the ring's slots (refills); more CTAs
than SMs; ragged N (not a multiple of 16 or of 4, fewer rows than one tile,
fewer rows than CTAs) and ragged M."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits
from tests.test_gpu_parity import DEV, _gemm_case, _np_bf16, assert_gemm_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [
    (1, 1, 256), (2, 3, 256), (5, 17, 512), (8, 100, 768), (3, 333, 1024),
    (7, 1000, 1536), (8, 4099, 2048), (4, 300, 4352), (1, 260, 8192), (6, 150, 7168),
    (9, 5, 256), (16, 333, 1024), (12, 1000, 1536), (15, 2049, 2048), (16, 260, 4352),
    (10, 300, 7168), (17, 50, 256), (24, 777, 1024), (31, 2049, 1536), (32, 129, 4352),
    (20, 300, 7168), (32, 64, 4096),
    (2, 9472, 8192),      # 4 tiles x 2 passes per CTA: slots refilled from the ring
    (3, 20000, 512),      # more CTAs than SMs (24 row quads each at most)
    (1, 14212, 256),      # just past one wave of 96-row CTAs
    (16, 9472, 8192),     # two column tiles: 4 tiles x 2 passes, ring refills
    (24, 9472, 8192),
    (13, 20000, 512),     # more CTAs than SMs
    (29, 20000, 2304),
    (32, 14212, 256),
    (9, 12288, 4096), (17, 12288, 4096), (32, 12288, 4096),   # the decode layer
])
def test_gemv_shapes(M, N, K):
    X, Wq, S, Y = _gemm_case(M, N, K, seed=M * 31 + N + K)
    _, R = oracle.w4a16_gemm(X, Wq, S)
    assert_gemm_close(Y, R, f"M={M} N={N} K={K}")


def test_gemv_laplace_weights():
    X, Wq, S, Y = _gemm_case(16, 1536, 2048, seed=3, w_dist="laplace")
    _, R = oracle.w4a16_gemm(X, Wq, S)
    assert_gemm_close(Y, R, "laplace")


@pytest.mark.parametrize("N,K,MB", [(256, 256, 8), (200, 1536, 8), (120, 4096, 8),
                                    (40, 4352, 5), (100, 2048, 16), (130, 4352, 32),
                                    (70, 2560, 27)])
def test_gemv_one_hot_exact(N, K, MB):
    """X = rows of the identity: Y[m, n] = dq(W)[n, k0 + m] exactly (one
    nonzero product per output: checks the fragment K order against the
    activation order, the row swizzle and the scale of every group)."""
    W = synth.normal_bf16((N, K), 0.02, seed=N + K, outlier_frac=0.01)
    Wq, S = oracle.quantize_pack(bits(W))
    Wdq = oracle.dequant(Wq, S)
    Wq_d, S_d = torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
    for m0 in range(0, K, MB * 7):
        M = min(MB, K - m0)
        X = torch.zeros((M, K), dtype=torch.bfloat16)
        X[torch.arange(M), m0 + torch.arange(M)] = 1.0
        Y = bits(w4.gemm(X.to(DEV), Wq_d, S_d))
        want = Wdq[:, m0:m0 + M].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch N={N} K={K} m0={m0}: {bad[:8].tolist()}")
    w4.w4_device_status()


@pytest.mark.parametrize("M", [5, 8])
def test_gemv_deterministic_and_no_workspace(M):
    N, K = 4096 + 12, 4096
    assert w4.w4a16_gemm_workspace_bytes(M, N, K) == 0
    X, Wq, S, Y1 = _gemm_case(M, N, K, seed=11)
    Xd, Wqd, Sd = _np_bf16(X).to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
    for _ in range(3):
        assert np.array_equal(bits(w4.gemm(Xd, Wqd, Sd)), Y1)
    w4.w4_device_status()


@pytest.mark.parametrize("M", [5, 11, 19])
def test_gemv_leaves_other_rows_of_y_alone(M):
    """Y is written only at [0, M) x [0, N): the rest of a larger flat buffer
    keeps its sentinel."""
    N, K = 333, 1024
    X, Wq, S, Y = _gemm_case(M, N, K, seed=21)
    flat = torch.full(((M + 3) * N,), -7.0, dtype=torch.bfloat16, device=DEV)
    w4.w4a16_gemm(_np_bf16(X).to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV),
                  flat[: M * N].view(M, N))
    w4.w4_device_status()
    assert np.array_equal(bits(flat[: M * N].view(M, N)), Y)
    assert bool((flat[M * N:] == -7.0).all())
