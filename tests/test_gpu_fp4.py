"""Parity of the micro-scaled FP4 path (MR-GPTQ / QuTLASS FP4 summary: MXFP4 =
E2M1 with a power-of-two scale per 32, NVFP4 = E2M1 with an E4M3 scale per 16
under an FP32 tensor scale) with the CPU oracle: quantizers and dequant bit for
bit, the W4A16 GEMM on FP4 weights within the GEMM tolerance and bit for bit on
one-hot activations.  The oracle keeps one code per byte; the GPU packs eight
per int32, low nibble first, so the tests pack the oracle's codes the same way."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits
from tests.test_gpu_parity import DEV, _np_bf16, assert_gemm_close

pytestmark = pytest.mark.gpu


def pack_codes(q: np.ndarray) -> np.ndarray:
    """[rows, K] uint8 codes (0..15) -> [rows, K/8] int32, element i of a word in bits 4i."""
    q = q.astype(np.uint32).reshape(q.shape[0], -1, 8)
    w = np.zeros(q.shape[:2], np.uint32)
    for i in range(8):
        w |= q[:, :, i] << np.uint32(4 * i)
    return w.view(np.int32)


def _dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _finite_bf16_patterns() -> np.ndarray:
    """Every finite BF16 bit pattern, padded to a multiple of 32 with zeros."""
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    b = b[(b & 0x7F80) != 0x7F80]
    pad = (-len(b)) % 32
    return np.concatenate([b, np.zeros(pad, np.uint16)])


def _edge_weights(N, K, seed, huge=True):
    """Ordinary groups next to the special cases; huge=False leaves out the
    group near the top of the BF16 range (its products overflow in a GEMM)."""
    W = synth.normal_bf16((N, K), 0.02, seed=seed, outlier_frac=0.01).clone()
    if N > 8 and K >= 256:
        W[0, 0:32] = 0.0                                                   # zero group
        W[1, 32:64] = 1e-39 * torch.linspace(-1, 1, 32).to(torch.bfloat16)  # subnormal amax
        if huge:
            W[2, 64:96] = (3e38 * torch.linspace(-1, 1, 32)).to(torch.bfloat16)  # near the top
        # every E2M1 rounding midpoint (and its negative) under amax 4 (MX: e = 0)
        mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0]
        W[3, 96:128] = torch.tensor(mids + [-m for m in mids] + mids + [-m for m in mids]
                                    ).to(torch.bfloat16)
        W[4, 128:160] = torch.tensor([0.5 * (i % 13 - 6) for i in range(32)]).to(torch.bfloat16)
        W[5, 160:192] = -0.001                                             # constant negative
    return W


# ---------------------------------------------------------------------------
# Dequant, exhaustive over codes and scales
# ---------------------------------------------------------------------------

def test_dequant_mxfp4_exhaustive():
    """Every code under every valid E8M0 exponent (0..254), including the
    subnormal and overflowing products."""
    E = np.arange(255, dtype=np.uint8).reshape(255, 1).repeat(2, axis=1)
    q = np.tile(np.arange(16, dtype=np.uint8), (255, 4))          # [255, 64]
    Wq = pack_codes(q)
    Wdq = bits(w4.dequant_mxfp4(_dev_u8(Wq), _dev_u8(E)))
    w4.w4_device_status()
    assert np.array_equal(Wdq, oracle.dequant_mxfp4(q, E))


@pytest.mark.parametrize("g", [1.0, 3.7e-5, 2.5e-3, 1e-40, 1e30, 0.3333333])
def test_dequant_nvfp4_exhaustive(g):
    """Every code under every valid E4M3 scale (both signs, 0x7F / 0xFF excluded)
    and tensor scales that underflow, overflow and round."""
    g = float(np.float32(g))
    sc = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    S = sc.reshape(-1, 1).repeat(4, axis=1)                        # [254, 4] (K = 64)
    q = np.tile(np.arange(16, dtype=np.uint8), (len(sc), 4))
    Wq = pack_codes(q)
    Wdq = bits(w4.dequant_nvfp4(_dev_u8(Wq), _dev_u8(S), g))
    w4.w4_device_status()
    assert np.array_equal(Wdq, oracle.dequant_nvfp4(q, S, g))


# ---------------------------------------------------------------------------
# Quantizers
# ---------------------------------------------------------------------------

def _check_mx(W_bits: np.ndarray):
    Wq, E = w4.quantize_pack_mxfp4(_np_bf16(W_bits).to(DEV))
    w4.w4_device_status()
    oq, oE = oracle.quantize_mxfp4(W_bits)
    assert np.array_equal(E.cpu().numpy(), oE)
    got, want = Wq.cpu().numpy(), pack_codes(oq)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} words differ, first [{r},{c}]: "
                             f"{got[r, c] & 0xFFFFFFFF:08x} vs {want[r, c] & 0xFFFFFFFF:08x}")


def _check_nv(W_bits: np.ndarray):
    Wq, S, g = w4.quantize_pack_nvfp4(_np_bf16(W_bits).to(DEV))
    w4.w4_device_status()
    oq, oS, og = oracle.quantize_nvfp4(W_bits)
    assert g.item() == og
    assert np.array_equal(S.cpu().numpy(), oS)
    got, want = Wq.cpu().numpy(), pack_codes(oq)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} words differ, first [{r},{c}]: "
                             f"{got[r, c] & 0xFFFFFFFF:08x} vs {want[r, c] & 0xFFFFFFFF:08x}")
    return Wq, S, g


def test_quantize_mxfp4_every_bf16_value():
    """All finite BF16 patterns: in bit order (groups of neighbouring values, every
    binade and the subnormals) and shuffled (small values under a large amax)."""
    b = _finite_bf16_patterns()
    _check_mx(b.reshape(-1, 256))
    rng = np.random.default_rng(0)
    _check_mx(rng.permutation(b).reshape(-1, 256))


def test_quantize_nvfp4_every_bf16_value():
    """As above, under the tensor scale that the whole pattern set implies (most
    group scales round to zero there), then the patterns below 2^-7 alone (a
    smaller tensor scale: the group scales spread over the E4M3 range)."""
    b = _finite_bf16_patterns()
    _check_nv(b.reshape(-1, 256))
    rng = np.random.default_rng(1)
    p = rng.permutation(b)
    _check_nv(p.reshape(-1, 256))
    small = b[(b & 0x7FFF) < 0x3C00]                 # |w| < 2^-7: g in the E4M3 subnormal reach
    small = small[: len(small) // 256 * 256]
    _check_nv(small.reshape(-1, 256))


def _nv_tie_groups(amax_t: float) -> np.ndarray:
    """Groups of 16 whose amax runs through every positive BF16 value up to
    amax_t (the tensor's amax, so g = fl32(amax_t / 2688)), each holding the
    E2M1 rounding midpoints of its expected step (E4M3(amax / 6), +-0.25 ..
    +-5 of it) and a zero; rows of 16 groups, zero-padded."""
    vals = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    vals = vals[vals <= amax_t]
    # torch's E4M3 conversion does not saturate: clamp at 448 first
    step = torch.from_numpy(np.minimum(vals / np.float32(6.0), np.float32(448.0)))
    step = step.to(torch.float8_e4m3fn).float().numpy()
    tq = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    el = step[:, None] * tq[None, :]
    grp = np.concatenate([vals[:, None], el, -el, np.zeros((len(vals), 1), np.float32)], axis=1)
    assert not np.any(grp.view(np.uint32) & 0xFFFF)          # all exact in BF16
    g_bits = (grp.view(np.uint32) >> 16).astype(np.uint16)
    pad = (-len(g_bits)) % 16
    g_bits = np.concatenate([g_bits, np.zeros((pad, 16), np.uint16)])
    return g_bits.reshape(-1, 256)


@pytest.mark.parametrize("amax_t", [2688.0, 2944.0])
def test_quantize_nvfp4_scale_and_code_ties(amax_t):
    """At g = 1 (tensor amax 2688) many group scales amax / 6 are exact E4M3
    midpoints and the elements exact E2M1 midpoints of their step: both
    decisions reach their exact FP64 path and must round ties to the even code.
    At g = fl32(2944 / 2688) the quotients fall near the midpoints instead."""
    W = _nv_tie_groups(amax_t)
    assert (W[:, :].view(np.uint16) & 0x7FFF).max() == np.float32(amax_t).view(np.uint32) >> 16
    _check_nv(W)


def test_quantize_nvfp4_row_scales_span_e4m3():
    """Rows scaled by 2^0 .. 2^-40 under one tensor scale: group scales run
    through every E4M3 binade, the subnormals and zero."""
    W = synth.normal_bf16((41, 512), 1.0, seed=8).float()
    W = W * torch.pow(2.0, -torch.arange(41, dtype=torch.float32)).reshape(-1, 1)
    _check_nv(bits(W.to(torch.bfloat16)))
    _check_mx(bits(W.to(torch.bfloat16)))


@pytest.mark.parametrize("rows,K", [(1, 32), (9, 256), (300, 640), (1000, 4096), (4097, 256)])
def test_quantize_fp4_edge_weights(rows, K):
    W = bits(_edge_weights(rows, K, seed=rows + K))
    _check_mx(W)
    _check_nv(W)


def test_quantize_fp4_zero_tensor():
    W = np.zeros((4, 64), np.uint16)
    _check_mx(W)
    Wq, S, g = _check_nv(W)
    assert g.item() == 1.0


def test_nvfp4_tensor_scale_odd_length():
    """The tensor amax sees a last odd element."""
    W = synth.normal_bf16((1, 1001), 0.02, seed=5).reshape(-1)
    W[1000] = 7.0
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    w4.w4_nvfp4_tensor_scale(W.to(DEV), g)
    assert g.item() == float(np.float32(7.0) / np.float32(2688.0))


@pytest.mark.parametrize("where", [0, 3, 500, 1998])
def test_nvfp4_tensor_scale_unaligned_views(where):
    """Views starting 4, 8 and 12 bytes past a 16-byte boundary: the amax pass
    reads the pairs before the first boundary and after the last whole 16
    bytes one word at a time; the largest value sits in the head, the middle
    or the ragged end."""
    base = synth.normal_bf16((1, 4096), 0.02, seed=6).reshape(-1).to(DEV)
    for off in (2, 4, 6):
        W = base[off:off + 2002]
        W[where] = -5.0
        g = torch.empty(1, dtype=torch.float32, device=DEV)
        w4.w4_nvfp4_tensor_scale(W, g)
        assert g.item() == float(np.float32(5.0) / np.float32(2688.0)), (off, where)
        W[where] = 0.0


def test_fp4_quantize_layer_shape():
    """The decode layer's weights (12288 x 4096): every output compared."""
    W = bits(synth.normal_bf16((12288, 4096), 0.02, seed=2, outlier_frac=0.001))
    _check_mx(W)
    _check_nv(W)


# ---------------------------------------------------------------------------
# GEMM on FP4 weights
# ---------------------------------------------------------------------------

def _mx_weights(N, K, seed):
    oq, oE = oracle.quantize_mxfp4(bits(_edge_weights(N, K, seed, huge=False)))
    return oq, oE, _dev_u8(pack_codes(oq)), _dev_u8(oE)


def _nv_weights(N, K, seed):
    oq, oS, og = oracle.quantize_nvfp4(bits(_edge_weights(N, K, seed, huge=False)))
    return oq, oS, og, _dev_u8(pack_codes(oq)), _dev_u8(oS)


# 1..8 rows with K % 512 == 0 take the warp-level decode kernel (one and
# several passes over K, ring refills, more CTAs than SMs, ragged N); 9..64
# rows with K % 256 == 0 the 256-wide decode tiles; the others the 64-wide
# tensor-memory tile
SHAPES = [(1, 1, 32), (1, 300, 4096), (5, 100, 128), (64, 300, 640), (65, 257, 256),
          (300, 1000, 1024), (512, 1024, 2048), (3, 129, 96), (8, 4099, 2048), (7, 1000, 1536),
          (2, 9472, 8192), (3, 20000, 512), (1, 14212, 512), (4, 37, 4608), (16, 300, 4096),
          (9, 1000, 1024), (32, 4099, 2048), (64, 129, 768), (24, 12288, 4096),
          (17, 20000, 512)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_mxfp4_shapes(M, N, K):
    oq, oE, Wq, E = _mx_weights(N, K, seed=M + N + K)
    X = synth.normal_bf16((M, K), 1.0, seed=M + 3)
    Y = bits(w4.gemm_mxfp4(X.to(DEV), Wq, E))
    w4.w4_device_status()
    _, R = oracle.gemm(bits(X), oracle.dequant_mxfp4(oq, oE))
    assert_gemm_close(Y, R, f"mxfp4 M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_nvfp4_shapes(M, N, K):
    oq, oS, og, Wq, S = _nv_weights(N, K, seed=M + N + K)
    X = synth.normal_bf16((M, K), 1.0, seed=M + 4)
    Y = bits(w4.gemm_nvfp4(X.to(DEV), Wq, S, og))
    w4.w4_device_status()
    _, R = oracle.gemm(bits(X), oracle.dequant_nvfp4(oq, oS, og))
    assert_gemm_close(Y, R, f"nvfp4 M={M} N={N} K={K}")


def _one_hot_check(run, Wdq, K, MB=64):
    for m0 in range(0, K, MB):
        X = torch.zeros((MB, K), dtype=torch.bfloat16)
        X[torch.arange(MB), m0 + torch.arange(MB)] = 1.0
        Y = bits(run(X.to(DEV)))
        want = Wdq[:, m0:m0 + MB].T
        if not np.array_equal(Y, want):
            bad = np.argwhere(Y != want)
            raise AssertionError(f"one-hot mismatch at m0={m0}: {bad[:8].tolist()}")


def test_gemm_fp4_one_hot_exact():
    """X = identity rows: Y[m, n] = Wdq[n, m] bit for bit for both formats
    (finite products only: a one-hot row reproduces an overflowing weight as inf)."""
    N, K = 200, 256
    oq, oE, Wq, E = _mx_weights(N, K, seed=11)
    _one_hot_check(lambda X: w4.gemm_mxfp4(X, Wq, E), oracle.dequant_mxfp4(oq, oE), K)
    oq, oS, og, Wq, S = _nv_weights(N, K, seed=12)
    _one_hot_check(lambda X: w4.gemm_nvfp4(X, Wq, S, og), oracle.dequant_nvfp4(oq, oS, og), K)
    w4.w4_device_status()


def test_gemm_fp4_one_hot_exact_decode_kernel():
    """The same with 8-row one-hot blocks, which the warp-level decode kernel
    takes (K % 512 == 0): every code position of the natural-order unpack
    meets its activation."""
    N, K = 120, 1024
    oq, oE, Wq, E = _mx_weights(N, K, seed=13)
    _one_hot_check(lambda X: w4.gemm_mxfp4(X, Wq, E), oracle.dequant_mxfp4(oq, oE), K, MB=8)
    oq, oS, og, Wq, S = _nv_weights(N, K, seed=14)
    _one_hot_check(lambda X: w4.gemm_nvfp4(X, Wq, S, og), oracle.dequant_nvfp4(oq, oS, og), K,
                   MB=8)
    w4.w4_device_status()


@pytest.mark.parametrize("M", [1, 8, 16, 2048])
def test_gemm_fp4_layer_shape_sampled(M):
    """The decode layer's weight (12288 x 4096) at 1, 8, 16 and 2048 tokens;
    the oracle checks up to 12 rows of Y spread over M."""
    N, K = 12288, 4096
    W = bits(synth.normal_bf16((N, K), 0.02, seed=6, outlier_frac=0.001))
    X = synth.normal_bf16((M, K), 1.0, seed=7)
    rows = torch.unique(torch.linspace(0, M - 1, 12).long())
    oq, oE = oracle.quantize_mxfp4(W)
    Y = w4.gemm_mxfp4(X.to(DEV), _dev_u8(pack_codes(oq)), _dev_u8(oE))
    _, R = oracle.gemm(bits(X[rows]), oracle.dequant_mxfp4(oq, oE))
    assert_gemm_close(bits(Y[rows.to(DEV)]), R, f"mxfp4 layer M={M}")
    oq, oS, og = oracle.quantize_nvfp4(W)
    Y = w4.gemm_nvfp4(X.to(DEV), _dev_u8(pack_codes(oq)), _dev_u8(oS), og)
    _, R = oracle.gemm(bits(X[rows]), oracle.dequant_nvfp4(oq, oS, og))
    assert_gemm_close(bits(Y[rows.to(DEV)]), R, f"nvfp4 layer M={M}")
    w4.w4_device_status()
