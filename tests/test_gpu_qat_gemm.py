"""Parity of the QAT GEMMs with fake quantization fused into the weight
prologue with the CPU oracle: the forward w4_qat_gemm, Y = X . fake_quant(W)^T,
and the input gradient w4_qat_gemm_dx, dX = dY . fake_quant(W).  The oracle
materializes fake_quant(W) and multiplies; the GPU never writes it."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits
from tests.test_gpu_parity import DEV, _np_bf16, assert_gemm_close

pytestmark = pytest.mark.gpu


def _case(M, N, K, seed, outliers=0.001):
    W = synth.normal_bf16((N, K), 0.02, seed=seed, outlier_frac=outliers)
    X = synth.normal_bf16((M, K), 1.0, seed=seed + 1)
    Y = bits(w4.qat_gemm(X.to(DEV), W.to(DEV)))
    w4.w4_device_status()
    Wdq, _ = oracle.fake_quant(bits(W))
    _, R = oracle.gemm(bits(X), Wdq)
    return Y, R


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (5, 100, 128), (64, 300, 640), (65, 257, 256),
                                   (300, 1000, 1024), (512, 1024, 2048), (3, 129, 4096)])
def test_qat_gemm_shapes(M, N, K):
    Y, R = _case(M, N, K, seed=M + N + K)
    assert_gemm_close(Y, R, f"qat M={M} N={N} K={K}")


def test_qat_gemm_one_hot_exact_with_edge_groups():
    """X = identity rows: Y[m, n] = fake_quant(W)[n, m] bit for bit, on weights
    with zero groups, subnormal-scale groups and huge values (the exact
    division path of the in-prologue QDQ) next to ordinary ones."""
    N, K = 200, 256
    W = synth.normal_bf16((N, K), 0.02, seed=9, outlier_frac=0.01).clone()
    W[3, 0:32] = 0.0                                        # amax 0 -> s = +0
    W[4, 32:64] = 1e-39                                     # subnormal scale
    W[5, 64:96] = torch.linspace(-3e30, 3e30, 32).to(torch.bfloat16)   # huge
    W[6, 96:128] = torch.tensor([0.5 * (i % 3 - 1) for i in range(32)]).to(torch.bfloat16)  # ties
    Wd = W.to(DEV)
    Wdq, _ = oracle.fake_quant(bits(W))
    for m0 in range(0, K, 64):
        X = torch.zeros((64, K), dtype=torch.bfloat16)
        X[torch.arange(64), m0 + torch.arange(64)] = 1.0
        Y = bits(w4.qat_gemm(X.to(DEV), Wd))
        want = Wdq[:, m0:m0 + 64].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch at m0={m0}: {bad[:8].tolist()}")
    w4.w4_device_status()


def test_qat_gemm_one_hot_subnormal_scales():
    """One-hot X on groups with subnormal scales, where the clamp to [-8, 7]
    fires: the in-prologue QDQ gives fake_quant(W) bit for bit."""
    from tests.test_gpu_parity import _subnormal_scale_groups
    G = _subnormal_scale_groups()
    rows = G.shape[0] // 8
    Wb = np.ascontiguousarray(G[: rows * 8].reshape(rows, 256))
    Wdq, _ = oracle.fake_quant(Wb)
    Wd = _np_bf16(Wb).to(DEV)
    K = 256
    for m0 in range(0, K, 64):
        X = torch.zeros((64, K), dtype=torch.bfloat16)
        X[torch.arange(64), m0 + torch.arange(64)] = 1.0
        Y = bits(w4.qat_gemm(X.to(DEV), Wd))
        want = Wdq[:, m0:m0 + 64].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch at m0={m0}: {bad[:8].tolist()}")
    w4.w4_device_status()


def test_qat_gemm_layer_shape_sampled():
    """A QAT-stack layer shape (W[12288, 4096]) at 2048 tokens; the oracle checks
    16 rows of Y spread over M (every weight group enters every checked element)."""
    N, K, M = 12288, 4096, 2048
    W = synth.normal_bf16((N, K), 0.02, seed=0, index=1, device=DEV, outlier_frac=0.001)
    X = synth.normal_bf16((M, K), 1.0, seed=0, index=2, device=DEV)
    Y = w4.qat_gemm(X, W)
    w4.w4_device_status()
    rows = torch.linspace(0, M - 1, 16).long()
    Wdq, _ = oracle.fake_quant(bits(W.cpu()))
    _, R = oracle.gemm(bits(X[rows].cpu()), Wdq)
    assert_gemm_close(bits(Y[rows]), R, "qat layer sampled")


def test_qat_gemm_matches_fake_quant_then_gemm():
    """The fused path and the unfused one (w4_fake_quant, then the same product
    from the materialized Wdq through the oracle) agree within GEMM tolerance,
    and the fused path is deterministic."""
    M, N, K = 128, 512, 1024
    W = synth.normal_bf16((N, K), 0.02, seed=4)
    X = synth.normal_bf16((M, K), 1.0, seed=5)
    Xd, Wd = X.to(DEV), W.to(DEV)
    Y1 = bits(w4.qat_gemm(Xd, Wd))
    Y2 = bits(w4.qat_gemm(Xd, Wd))
    assert np.array_equal(Y1, Y2)
    Wdq_gpu = bits(w4.fake_quant(Wd))
    _, R = oracle.gemm(bits(X), Wdq_gpu)
    assert_gemm_close(Y1, R, "fused vs materialized")


# ---------------------------------------------------------------------------
# Input gradient with the fused QDQ: dX = dY . fake_quant(W)
# ---------------------------------------------------------------------------

def _dx_case(M, N, K, seed, outliers=0.001):
    W = synth.normal_bf16((N, K), 0.02, seed=seed, outlier_frac=outliers)
    dY = synth.normal_bf16((M, N), 1.0, seed=seed + 1)
    dX = bits(w4.qat_gemm_dx(dY.to(DEV), W.to(DEV)))
    w4.w4_device_status()
    Wdq, _ = oracle.fake_quant(bits(W))
    _, R = oracle.gemm(bits(dY), np.ascontiguousarray(Wdq.T))
    return dX, R


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (5, 104, 128), (64, 320, 640), (65, 264, 256),
                                   (300, 1000, 1024), (512, 1024, 2048), (3, 136, 4096),
                                   (17, 4096, 192)])
def test_qat_gemm_dx_shapes(M, N, K):
    """Ragged token tiles, a partial last 64-wide block of N and a partial
    last 128-row tile of K."""
    dX, R = _dx_case(M, N, K, seed=M + N + K)
    assert_gemm_close(dX, R, f"qat dx M={M} N={N} K={K}")


def test_qat_gemm_dx_one_hot_exact_with_edge_groups():
    """dY = identity rows: dX[m, :] = fake_quant(W)[n0 + m, :] bit for bit, on
    weights with zero, subnormal-scale, huge and tie groups."""
    N, K = 192, 256
    W = synth.normal_bf16((N, K), 0.02, seed=9, outlier_frac=0.01).clone()
    W[3, 0:32] = 0.0
    W[4, 32:64] = 1e-39
    W[5, 64:96] = torch.linspace(-3e30, 3e30, 32).to(torch.bfloat16)
    W[6, 96:128] = torch.tensor([0.5 * (i % 3 - 1) for i in range(32)]).to(torch.bfloat16)
    Wd = W.to(DEV)
    Wdq, _ = oracle.fake_quant(bits(W))
    for n0 in range(0, N, 64):
        dY = torch.zeros((64, N), dtype=torch.bfloat16)
        dY[torch.arange(64), n0 + torch.arange(64)] = 1.0
        dX = bits(w4.qat_gemm_dx(dY.to(DEV), Wd))
        want = Wdq[n0:n0 + 64, :]
        if not np.array_equal(dX, want):
            bad = np.argwhere(dX != want)
            raise AssertionError(f"one-hot mismatch at n0={n0}: {bad[:8].tolist()}")
    w4.w4_device_status()


def test_qat_gemm_dx_layer_shape_sampled():
    """A QAT-stack layer (W[12288, 4096]) at 2048 tokens: dX [2048, 4096]; the
    oracle checks 12 rows (every weight enters every checked element)."""
    N, K, M = 12288, 4096, 2048
    W = synth.normal_bf16((N, K), 0.02, seed=0, index=1, device=DEV, outlier_frac=0.001)
    dY = synth.normal_bf16((M, N), 1.0, seed=0, index=3, device=DEV)
    dX = w4.qat_gemm_dx(dY, W)
    w4.w4_device_status()
    rows = torch.linspace(0, M - 1, 12).long()
    Wdq, _ = oracle.fake_quant(bits(W.cpu()))
    _, R = oracle.gemm(bits(dY[rows.to(DEV)].cpu()), np.ascontiguousarray(Wdq.T))
    assert_gemm_close(bits(dX[rows.to(DEV)]), R, "qat dx layer sampled")


def test_qat_gemm_dx_matches_fake_quant_then_gemm_and_is_deterministic():
    M, N, K = 128, 512, 1024
    W = synth.normal_bf16((N, K), 0.02, seed=4)
    dY = synth.normal_bf16((M, N), 1.0, seed=6)
    dYd, Wd = dY.to(DEV), W.to(DEV)
    a = bits(w4.qat_gemm_dx(dYd, Wd))
    b = bits(w4.qat_gemm_dx(dYd, Wd))
    assert np.array_equal(a, b)
    Wdq_gpu = bits(w4.fake_quant(Wd))
    _, R = oracle.gemm(bits(dY), np.ascontiguousarray(Wdq_gpu.T))
    assert_gemm_close(a, R, "fused dx vs materialized")


def test_qat_gemms_one_hot_several_token_tiles():
    """More than 256 tokens run several 256-token work items per weight tile
    (the forward with the QDQ written back over the weight tile, both with two
    accumulator sets): one-hot rows give fake_quant(W) bit for bit across the
    items and the ragged end."""
    N, K, M = 384, 512, 320
    W = synth.normal_bf16((N, K), 0.02, seed=17, outlier_frac=0.01).clone()
    W[7, 32:64] = 1e-39                                   # subnormal scale
    W[9, 64:96] = 0.0
    Wdq, _ = oracle.fake_quant(bits(W))
    Wd = W.to(DEV)
    X = torch.zeros((M, K), dtype=torch.bfloat16)
    X[torch.arange(M), torch.arange(M)] = 1.0
    Y = bits(w4.qat_gemm(X.to(DEV), Wd))                  # Y[m, n] = Wdq[n, m]
    assert np.array_equal(Y, Wdq[:, :M].T)
    dY = torch.zeros((M, N), dtype=torch.bfloat16)
    dY[torch.arange(M), torch.arange(M)] = 1.0
    dX = bits(w4.qat_gemm_dx(dY.to(DEV), Wd))             # dX[m, :] = Wdq[m, :]
    assert np.array_equal(dX, Wdq[:M, :])
    w4.w4_device_status()


@pytest.mark.parametrize("M", [1, 64, 200, 256])
def test_qat_gemms_split_matches_unsplit(M):
    """Up to 256 tokens the QAT GEMMs cut the (row tile, k-block) units over
    the SMs (workspace): same product as the unsplit schedule within the GEMM
    tolerance, deterministic, counters left zero, and against the oracle."""
    N, K = 4096, 4096
    assert w4.w4_qat_gemm_workspace_bytes(M, N, K) > 0          # 32 row tiles < SMs / 2
    W = synth.normal_bf16((N, K), 0.02, seed=M, outlier_frac=0.001)
    X = synth.normal_bf16((M, K), 1.0, seed=M + 1)
    dY = synth.normal_bf16((M, N), 1.0, seed=M + 2)
    Wd, Xd, dYd = W.to(DEV), X.to(DEV), dY.to(DEV)
    ws = torch.zeros(max(w4.w4_qat_gemm_workspace_bytes(M, N, K), 256), dtype=torch.uint8,
                     device=DEV)
    Wdq, _ = oracle.fake_quant(bits(W))
    Y1, Y2 = bits(w4.qat_gemm(Xd, Wd, ws=ws)), bits(w4.qat_gemm(Xd, Wd, ws=ws))
    D1, D2 = bits(w4.qat_gemm_dx(dYd, Wd, ws=ws)), bits(w4.qat_gemm_dx(dYd, Wd, ws=ws))
    w4.w4_device_status()
    assert np.array_equal(Y1, Y2) and np.array_equal(D1, D2)
    assert int(ws[:4096].count_nonzero()) == 0, "split counters not reset"
    _, R = oracle.gemm(bits(X), Wdq)
    assert_gemm_close(Y1, R, f"qat split M={M}")
    assert_gemm_close(bits(w4.qat_gemm(Xd, Wd, ws=None)), R, f"qat unsplit M={M}")
    _, Rd = oracle.gemm(bits(dY), np.ascontiguousarray(Wdq.T))
    assert_gemm_close(D1, Rd, f"qat dx split M={M}")
    assert_gemm_close(bits(w4.qat_gemm_dx(dYd, Wd, ws=None)), Rd, f"qat dx unsplit M={M}")
