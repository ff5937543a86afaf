"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Integer and byte outputs (codes, scales, packed words, dequantized BF16, STE,
moe_align) must match bit for bit.  GEMM outputs Y are compared with the
oracle's FP32-accumulated sums R:  max|Y - R| / max|R| <= 1e-2 and, element by
element, |Y - R| <= 1e-2 |R| + 1e-3 max|R|  (BF16 output rounding alone gives
about 2^-9 relative).
"""
import json
import os

import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits

pytestmark = pytest.mark.gpu

DEV = "cuda"
GOLD = os.path.join(os.path.dirname(__file__), "golden")
REL_TOL = 1e-2


def _np_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def assert_gemm_close(Y_bits: np.ndarray, R: np.ndarray, what: str):
    y = (Y_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = R.astype(np.float64)
    scale = np.abs(r).max()
    err = np.abs(y - r)
    assert scale > 0
    assert err.max() / scale <= REL_TOL, f"{what}: max err / max|R| = {err.max() / scale:.3e}"
    bad = err > REL_TOL * np.abs(r) + 1e-3 * scale
    assert not bad.any(), f"{what}: {bad.sum()} elements outside tolerance, e.g. {np.argwhere(bad)[:5]}"


# ---------------------------------------------------------------------------
# Quantizers
# ---------------------------------------------------------------------------

def _check_quantizers(W_cpu_bf16: torch.Tensor):
    Wb = bits(W_cpu_bf16)
    Wq_o, S_o = oracle.quantize_pack(Wb)
    Wdq_o, S2_o = oracle.fake_quant(Wb)
    W = W_cpu_bf16.to(DEV)
    Wq, S = w4.quantize_pack(W)
    Wdq, S2 = w4.fake_quant(W, want_scales=True)
    D = w4.dequant(Wq, S)
    w4.w4_device_status()
    assert np.array_equal(bits(S), S_o), "scales"
    assert np.array_equal(Wq.cpu().numpy(), Wq_o), "packed words"
    assert np.array_equal(bits(S2), S2_o), "fake-quant scales"
    assert np.array_equal(bits(Wdq), Wdq_o), "fake-quant output"
    assert np.array_equal(bits(D), Wdq_o), "dequant of export"


def test_hand_groups_on_gpu():
    g = json.load(open(os.path.join(GOLD, "hand_groups.json")))
    A = torch.tensor(g["group_A"]["inputs"], dtype=torch.float32).to(torch.bfloat16)
    B = ((torch.arange(32, dtype=torch.float32) - 16) * torch.tensor(0.001)).to(torch.bfloat16)
    W = torch.stack([A, B]).to(DEV)
    Wq, S = w4.quantize_pack(W)
    assert [hex(int(x)) for x in bits(S).ravel()] == ["0x3f80", "0x3b16"]
    words = _u32(Wq)
    assert [int(x) for x in words[0]] == [int(h, 16) for h in g["group_A"]["words"]]
    assert [int(x) for x in words[1]] == [int(h, 16) for h in g["group_B"]["words"]]


@pytest.mark.parametrize("rows,K", [(1, 32), (3, 64), (17, 96), (5, 1024), (257, 320),
                                    (1024, 1024), (333, 4096)])
def test_quantizers_ragged(rows, K):
    _check_quantizers(synth.normal_bf16((rows, K), 0.02, seed=rows + K, outlier_frac=0.001))


def test_quantizers_laplace_and_ties():
    _check_quantizers(synth.laplace_bf16((512, 2048), 0.015, seed=3))
    # tie-heavy: every group has amax 7 * 2^e and entries on the half-integer grid
    rng = np.random.default_rng(5)
    halves = rng.integers(-14, 15, size=(256, 1024)).astype(np.float32) / 2.0
    halves[:, ::32] = 7.0
    exps = rng.integers(-20, 20, size=(256, 1)).astype(np.float32)
    W = torch.from_numpy(halves * np.exp2(exps)).to(torch.bfloat16)
    _check_quantizers(W)


def test_quantizers_edge_scales():
    rows = []
    z = np.zeros(32, np.uint16)
    rows.append(z)                                          # all zero
    t = z.copy(); t[0] = 0x0001; t[5] = 0x8001; rows.append(t)   # amax/7 rounds to 0
    t = z.copy(); t[:] = 0x0080; t[3] = 0x00E0; rows.append(t)   # subnormal scale path
    t = z.copy(); t[:] = 0x0380; rows.append(t)                  # tiny normal scale
    t = np.full(32, 0x7F00, np.uint16); t[1::2] |= 0x8000; rows.append(t)  # huge values
    t = np.arange(32, dtype=np.uint16) | 0x8000; rows.append(t)  # negative subnormals
    t = z.copy(); t[7] = 0x8000; t[9] = 0x3F80; rows.append(t)   # -0.0 entries
    W = _np_bf16(np.stack(rows))
    _check_quantizers(W)


def _subnormal_scale_groups() -> np.ndarray:
    """Groups whose BF16 scale is subnormal (amax below 7 * 2^-126): there the
    scale carries 1..7 significant bits, so |w / s| reaches 8 and more and the
    clamp to [-8, 7] decides the code ("量化基础" §1.3, INT4 = [-8, 7])."""
    g = []
    ramp = np.arange(32, dtype=np.uint16)
    g.append(ramp)                                   # +0x0000 .. +0x001F
    g.append(ramp | 0x8000)                          # -0x0000 .. -0x001F
    t = np.zeros(32, np.uint16); t[0] = 0x000A; g.append(t)      # s = 2^-133, w/s = 10
    t = np.zeros(32, np.uint16); t[17] = 0x800A; g.append(t)
    # every positive subnormal amax heads a ramp of both signs, and its negation
    for a in range(0x0001, 0x0080):
        v = np.linspace(a, 0, 32).round().astype(np.uint16)
        v[1::2] |= 0x8000
        v[0] = a
        g.append(v)
        g.append(v ^ 0x8000)
    return np.stack(g)


def test_quantizers_subnormal_scales_clamp():
    G = _subnormal_scale_groups()
    # the groups really reach past the INT4 range before the clamp
    w = (G.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    _, S = oracle.quantize(G)
    s = (S.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(s > 0, w / np.where(s > 0, s, 1.0), 0.0)
    assert np.rint(y).max() >= 8 and np.rint(y).min() <= -9
    q, _ = oracle.quantize(G)
    assert q.max() == 7 and q.min() == -8
    _check_quantizers(_np_bf16(G))
    # the same groups as rows of a wider matrix (several groups per row)
    rows = G.shape[0] // 8
    _check_quantizers(_np_bf16(G[: rows * 8].reshape(rows, 256)))


def test_quantizers_decode_weight_full():
    _check_quantizers(synth.Decode().weight())


def test_quantizers_qat_stack_sampled():
    """Config 5 (48 x (12288x4096 + 4096x12288)): layer 0 checked in full, the
    other layers on 64 rows each (generated on the device, copied back)."""
    cfg = synth.QATStack()
    for layer in range(cfg.layers):
        for which in range(2):
            W = cfg.weight(layer, which, device=DEV)
            Wq, S = w4.quantize_pack(W)
            Wdq = w4.fake_quant(W)
            rows = W.shape[0]
            sel = slice(None) if layer == 0 else torch.linspace(0, rows - 1, 64).long()
            Wb = bits(W[sel])
            Wq_o, S_o = oracle.quantize_pack(Wb)
            Wdq_o, _ = oracle.fake_quant(Wb)
            assert np.array_equal(Wq[sel].cpu().numpy(), Wq_o), (layer, which)
            assert np.array_equal(bits(S[sel]), S_o), (layer, which)
            assert np.array_equal(bits(Wdq[sel]), Wdq_o), (layer, which)
            del W, Wq, S, Wdq
    w4.w4_device_status()


def test_ste_backward():
    g = synth.normal_bf16((4096, 1031), 1e-3, seed=9).to(DEV)    # odd size: tail copy
    dW = torch.empty_like(g)
    w4.w4_ste_backward(g, dW)
    assert torch.equal(g.view(torch.int16), dW.view(torch.int16))
    w4.w4_ste_backward(g, g)                                      # aliased: no-op
    W = synth.normal_bf16((64, 256), 0.02, seed=1).to(DEV).requires_grad_(True)
    out = w4.FakeInt4STE.apply(W)
    grad = torch.randn_like(out)
    out.backward(grad)
    assert torch.equal(W.grad.view(torch.int16), grad.view(torch.int16))


def test_16_byte_aligned_buffers():
    """Buffers aligned to 16 but not 32 bytes take the 16-byte load/store kernels;
    results are identical to the oracle either way."""
    n = 4099 * 9                                   # not a multiple of 16: tail copy
    src = synth.normal_bf16((n + 16,), 1e-3, seed=21).to(DEV)
    dst = torch.zeros(n + 16, dtype=torch.bfloat16, device=DEV)
    for so in (0, 8):
        for do in (0, 8):
            dst.zero_()
            w4.w4_ste_backward(src[so:so + n], dst[do:do + n])
            assert torch.equal(src[so:so + n].view(torch.int16), dst[do:do + n].view(torch.int16))
            assert not dst[:do].view(torch.int16).any() and not dst[do + n:].view(torch.int16).any()
    rows, K = 96, 512
    W_cpu = synth.laplace_bf16((rows, K), 0.02, seed=22)
    Wq_o, S_o = oracle.quantize_pack(bits(W_cpu))
    Wdq_o, _ = oracle.fake_quant(bits(W_cpu))
    buf = torch.zeros(rows * K + 8, dtype=torch.bfloat16, device=DEV)
    buf[8:] = W_cpu.reshape(-1).to(DEV)
    W = buf[8:].view(rows, K)                      # 16-byte but not 32-byte aligned
    assert W.data_ptr() % 32 == 16
    Wq, S = w4.quantize_pack(W)
    out = torch.zeros(rows * K + 8, dtype=torch.bfloat16, device=DEV)
    Wdq = out[8:].view(rows, K)
    w4.w4_fake_quant(W, Wdq)
    w4.w4_device_status()
    assert np.array_equal(Wq.cpu().numpy(), Wq_o)
    assert np.array_equal(bits(S), S_o)
    assert np.array_equal(bits(Wdq), Wdq_o)


def test_dequant_exhaustive_words():
    """Every code value at every nibble position, times a spread of scales."""
    rng = np.random.default_rng(1)
    words = rng.integers(-2**31, 2**31, size=(4096, 64), dtype=np.int64).astype(np.int32)
    words[0, :16] = np.array([np.uint32(v * 0x11111111).view(np.int32) for v in range(16)])
    S = rng.integers(0x0001, 0x7F00, size=(4096, 16)).astype(np.uint16)
    D = w4.dequant(torch.from_numpy(words).to(DEV), _np_bf16(S).to(DEV))
    assert np.array_equal(bits(D), oracle.dequant(words, S))


# ---------------------------------------------------------------------------
# W4A16 GEMM
# ---------------------------------------------------------------------------

def _gemm_case(M, N, K, seed, w_dist="normal"):
    if w_dist == "normal":
        W = synth.normal_bf16((N, K), 0.02, seed=seed, outlier_frac=0.001)
    else:
        W = synth.laplace_bf16((N, K), 0.015, seed=seed)
    X = synth.normal_bf16((M, K), 1.0, seed=seed + 1)
    Wq, S = oracle.quantize_pack(bits(W))
    Y = w4.gemm(X.to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV))
    w4.w4_device_status()
    return bits(X), Wq, S, bits(Y)


def test_gemm_one_hot_exact():
    """X = identity rows: Y[k, n] must equal dq(W)[n, k] exactly (checks the
    unpack indexing, the TMEM operand layout and the scale broadcast)."""
    for (N, K) in [(256, 256), (200, 512), (1024, 1024)]:
        W = synth.normal_bf16((N, K), 0.02, seed=N + K, outlier_frac=0.01)
        Wq, S = oracle.quantize_pack(bits(W))
        Wdq = oracle.dequant(Wq, S)
        Wq_d, S_d = torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
        for m0 in range(0, K, 64 if K > 256 else 16):
            M = min(64 if K > 256 else 16, K - m0)
            X = torch.zeros((M, K), dtype=torch.bfloat16)
            X[torch.arange(M), m0 + torch.arange(M)] = 1.0
            Y = bits(w4.gemm(X.to(DEV), Wq_d, S_d))
            want = Wdq[:, m0:m0 + M].T
            if not np.array_equal(Y, want):
                bad = np.argwhere(Y != want)
                raise AssertionError(f"one-hot mismatch N={N} K={K} m0={m0}: {bad[:8].tolist()}")


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (1, 8, 256), (3, 100, 96), (4, 1024, 1024),
                                   (17, 333, 512), (32, 4096, 1024), (64, 129, 768),
                                   (65, 300, 256), (300, 257, 320), (256, 1024, 2048)])
def test_gemm_small(M, N, K):
    X, Wq, S, Y = _gemm_case(M, N, K, seed=M * 7 + N)
    _, R = oracle.w4a16_gemm(X, Wq, S)
    assert_gemm_close(Y, R, f"M={M} N={N} K={K}")


def test_gemm_tiny_layer_config():
    cfg = synth.TinyLayer()
    X, W = cfg.activations(), cfg.weight()
    Wq, S = w4.quantize_pack(W.to(DEV))
    Y = bits(w4.gemm(X.to(DEV), Wq, S))
    _, R = oracle.w4a16_gemm(bits(X), Wq.cpu().numpy(), bits(S))
    assert_gemm_close(Y, R, "tiny layer")


_DECODE = {}


def _decode_weight():
    if "w" not in _DECODE:
        cfg = synth.Decode()
        _DECODE["w"] = oracle.quantize_pack(bits(cfg.weight()))
    return _DECODE["w"]


@pytest.mark.parametrize("M,split", [(1, False), (8, False), (16, True), (16, False),
                                     (32, True), (32, False), (64, True), (64, False)])
def test_gemm_decode_config(M, split):
    """Decode GEMV sweep: 1..8 rows take the warp-level MMA kernel (no
    workspace; `split` makes no difference there); 16..64 rows the
    tensor-memory kernel, with the stream-K split (workspace) and without."""
    cfg = synth.Decode()
    Wq, S = _decode_weight()
    X = cfg.activations(M)
    ws = "auto" if split else None
    assert (w4.w4a16_gemm_workspace_bytes(M, cfg.N, cfg.K) > 0) == (M > 8)
    Y = bits(w4.gemm(X.to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV), ws=ws))
    _, R = oracle.w4a16_gemm(bits(X), Wq, S)
    assert_gemm_close(Y, R, f"decode M={M} split={split}")


@pytest.mark.parametrize("M", [1, 8, 16, 32])
def test_gemm_reads_weights_the_previous_kernel_wrote(M):
    """The GEMMs may become resident (and warm L2 with their weight tiles)
    while the kernel before them on the stream still runs.  Here that kernel
    overwrites the packed weights and scales the GEMM reads, right after a GEMM
    on the old contents: the product must be that of the new weights."""
    N, K = 4096, 2048
    Wa = synth.normal_bf16((N, K), 0.02, seed=11).to(DEV)
    Wb = synth.normal_bf16((N, K), 0.5, seed=12).to(DEV)
    X = synth.normal_bf16((M, K), 1.0, seed=13).to(DEV)
    Wq = torch.empty((N, K // 8), dtype=torch.int32, device=DEV)
    S = torch.empty((N, K // 32), dtype=torch.bfloat16, device=DEV)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    for _ in range(3):
        w4.w4_quantize_pack(Wa, Wq, S)
        w4.w4a16_gemm(X, Wq, S, Y)
        w4.w4_quantize_pack(Wb, Wq, S)
        w4.w4a16_gemm(X, Wq, S, Y)
    w4.w4_device_status()
    oWq, oS = oracle.quantize_pack(bits(Wb.cpu()))
    assert np.array_equal(Wq.cpu().numpy(), oWq)
    _, R = oracle.w4a16_gemm(bits(X.cpu()), oWq, oS)
    assert_gemm_close(bits(Y), R, f"weights rewritten before the GEMM, M={M}")


def test_gemm_split_workspace_left_zero_and_deterministic():
    M, N, K = 16, 4096 + 200, 2048          # ragged last row tile, 8 k-blocks
    X, Wq, S, Y1 = _gemm_case(M, N, K, seed=5)
    need = w4.w4a16_gemm_workspace_bytes(M, N, K)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    Xd, Wqd, Sd = _np_bf16(X).to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
    outs = [bits(w4.gemm(Xd, Wqd, Sd, ws=ws)) for _ in range(3)]
    w4.w4_device_status()
    n_rt = (N + 127) // 128
    assert int(ws[: n_rt * 16].count_nonzero()) == 0, "split counters not reset"
    assert all(np.array_equal(o, outs[0]) for o in outs)
    _, R = oracle.w4a16_gemm(X, Wq, S)
    assert_gemm_close(outs[0], R, "split ragged")
    # the unsplit schedule gives the same product within tolerance
    Y0 = bits(w4.gemm(Xd, Wqd, Sd, ws=None))
    assert_gemm_close(Y0, R, "unsplit ragged")


def test_gemm_split_workspace_shared_across_shapes():
    """One zeroed workspace serves a sequence of split GEMMs with different
    row-tile counts: a call's parked partial sums never sit where a later call
    with more row tiles keeps its arrival counters."""
    M, K = 32, 2048
    ws = torch.zeros(w4.w4a16_gemm_workspace_bytes(M, 12288, K) + (1 << 20), dtype=torch.uint8,
                     device=DEV)
    for N in (4096, 9472, 12288, 640, 12288):
        X, Wq, S, _ = _gemm_case(M, N, K, seed=N)
        assert w4.w4a16_gemm_workspace_bytes(M, N, K) > 0
        Y = bits(w4.gemm(_np_bf16(X).to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV),
                         ws=ws))
        w4.w4_device_status()
        _, R = oracle.w4a16_gemm(X, Wq, S)
        assert_gemm_close(Y, R, f"shared workspace N={N}")


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_gemm_prefill_config_sampled(M):
    """Full-size prefill GEMM on the device; the oracle checks 24 rows of Y
    spread over M (every weight group still enters every checked element)."""
    cfg = synth.Prefill()
    W = cfg.weight(device=DEV)
    Wq, S = w4.quantize_pack(W)
    X = cfg.activations(M, device=DEV)
    Y = w4.gemm(X, Wq, S)
    w4.w4_device_status()
    rows = torch.linspace(0, M - 1, 24).long()
    _, R = oracle.w4a16_gemm(bits(X[rows]), Wq.cpu().numpy(), bits(S))
    assert_gemm_close(bits(Y[rows]), R, f"prefill M={M}")


def test_gemm_deterministic():
    X, Wq, S, Y1 = _gemm_case(300, 1000, 1024, seed=77)
    Y2 = bits(w4.gemm(_np_bf16(X).to(DEV), torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)))
    assert np.array_equal(Y1, Y2)


# ---------------------------------------------------------------------------
# MoE
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,topk,E,block", [(1, 1, 1, 16), (3, 2, 8, 16), (16, 8, 128, 16),
                                            (64, 8, 128, 32), (256, 8, 128, 64),
                                            (1000, 6, 64, 128), (5, 8, 1024, 256),
                                            (0, 8, 128, 16)])
def test_moe_align(T, topk, E, block):
    ids, _ = synth.routing(T, E, topk, seed=T + E) if T > 0 else (torch.zeros((0, topk), dtype=torch.int32), None)
    s_o, e_o, n_o = oracle.moe_align(ids.numpy(), E, block)
    s, e, n = w4.moe_align(ids.to(DEV), E, block)
    assert int(n.item()) == n_o
    assert np.array_equal(s.cpu().numpy(), s_o)
    assert np.array_equal(e.cpu().numpy(), e_o)


def test_moe_align_skewed_and_invalid_ids():
    rng = np.random.default_rng(0)
    ids = rng.integers(0, 3, size=(500, 4)).astype(np.int32)     # 3 of 16 experts
    ids[::7, 1] = -1
    ids[::11, 2] = 99                                            # out of range: skipped
    s_o, e_o, n_o = oracle.moe_align(ids, 16, 16)
    s, e, n = w4.moe_align(torch.from_numpy(ids).to(DEV), 16, 16)
    assert int(n.item()) == n_o
    assert np.array_equal(s.cpu().numpy(), s_o) and np.array_equal(e.cpu().numpy(), e_o)


_EXPERTS = {}


def _experts(E, N, K):
    """Per-expert packed weights (oracle export), cached across tests."""
    if (E, N, K) not in _EXPERTS:
        W = synth.normal_bf16((E, N, K), 0.02, seed=N + K)
        Wq = np.empty((E, N, K // 8), np.int32)
        S = np.empty((E, N, K // 32), np.uint16)
        for e in range(E):
            Wq[e], S[e] = oracle.quantize_pack(bits(W[e]))
        Wdq = np.stack([oracle.dequant(Wq[e], S[e]) for e in range(E)])
        _EXPERTS[(E, N, K)] = (Wq, S, Wdq)
    return _EXPERTS[(E, N, K)]


def _moe_case(T, block, N, K, E=128, topk=8, seed=0, down=False):
    ids, _ = synth.routing(T, E, topk, seed=seed + T)
    Wq, S, Wdq = _experts(E, N, K)
    rows = T * topk if down else T
    A = synth.normal_bf16((rows, K), 1.0, seed=seed + 2)
    a_row_div = 1 if down else topk
    s_d, e_d, n_d = w4.moe_align(ids.to(DEV), E, block)
    canary = torch.full((T * topk, N), 0x7FC1, dtype=torch.int16).view(torch.bfloat16).to(DEV)
    C = w4.moe_gemm(A.to(DEV), a_row_div, torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV),
                    s_d, e_d, n_d, block, T * topk, C=canary)
    w4.w4_device_status()
    s_o, e_o, n_o = oracle.moe_align(ids.numpy(), E, block)
    canary_np = np.full((T * topk, N), 0x7FC1, np.uint16)
    C_o, R = oracle.moe_gemm(bits(A), a_row_div, Wdq, s_o, e_o, n_o, T * topk, block,
                             C_init=canary_np)
    return bits(C), R, ids


@pytest.mark.parametrize("T,block", [(16, 16), (16, 32), (16, 64), (64, 16), (64, 32), (64, 64),
                                     (256, 16), (256, 32)])
def test_moe_gemm_gate_up(T, block):
    C, R, _ = _moe_case(T, block, N=3072, K=4096, seed=T)
    assert not np.any(C == 0x7FC1), "a real slot was left unwritten"
    assert_gemm_close(C, R, f"moe gate_up T={T} block={block}")


@pytest.mark.parametrize("T,block", [(16, 16), (64, 32), (256, 16), (256, 32)])
def test_moe_gemm_down(T, block):
    C, R, _ = _moe_case(T, block, N=4096, K=1536, seed=100 + T, down=True)
    assert_gemm_close(C, R, f"moe down T={T} block={block}")


@pytest.mark.parametrize("T,E,block", [(64, 8, 32), (40, 8, 64), (48, 16, 32)])
def test_moe_gemm_dense_routing(T, E, block):
    """Few experts, many slots each: 32-slot blocks that the routing fills
    (>= 16 slots per expert) run as 32-slot work items; wider or emptier blocks
    run as 16-slot sub-blocks with the all-padding ones skipped."""
    C, R, _ = _moe_case(T, block, N=700, K=1024, E=E, seed=7 * T + E)
    assert not np.any(C == 0x7FC1), "a real slot was left unwritten"
    assert_gemm_close(C, R, f"moe T={T} E={E} block={block}")


def test_moe_gemm_padding_rows_untouched():
    """Slots that no expert owns (routing ids out of range) keep the canary."""
    E, N, K, T, topk, block = 8, 256, 512, 10, 2, 16
    ids = torch.randint(0, E, (T, topk), generator=torch.Generator().manual_seed(3)).int()
    ids[0, 0] = -1
    ids[4, 1] = 50
    W = synth.normal_bf16((E, N, K), 0.02, seed=4)
    Wq = np.empty((E, N, K // 8), np.int32)
    S = np.empty((E, N, K // 32), np.uint16)
    for e in range(E):
        Wq[e], S[e] = oracle.quantize_pack(bits(W[e]))
    A = synth.normal_bf16((T, K), 1.0, seed=5)
    s_d, e_d, n_d = w4.moe_align(ids.to(DEV), E, block)
    canary = torch.full((T * topk, N), 0x7FC1, dtype=torch.int16).view(torch.bfloat16).to(DEV)
    C = bits(w4.moe_gemm(A.to(DEV), topk, torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV),
                         s_d, e_d, n_d, block, T * topk, C=canary))
    assert np.all(C[0] == 0x7FC1) and np.all(C[9] == 0x7FC1)
    assert not np.any(np.delete(C, [0, 9], axis=0) == 0x7FC1)
