"""Parity of the MoE layer glue on the GPU with the CPU oracle, through the C ABI:
router gating (softmax + top-k), the SiLU-gated product and the weighted top-k
combine, then one whole MoE layer (gating -> moe_align -> gate_up -> SiLU*up ->
down -> combine) checked stage by stage."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits
from tests.test_gpu_parity import DEV, _experts, _np_bf16, assert_gemm_close

pytestmark = pytest.mark.gpu


def _logits(T, E, seed):
    return np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)


@pytest.mark.parametrize("T,E,topk", [(1, 128, 8), (16, 128, 8), (256, 128, 8), (1000, 128, 8),
                                      (37, 8, 1), (64, 33, 33), (9, 256, 32), (5, 1, 1)])
def test_gate_topk(T, E, topk):
    logits = _logits(T, E, seed=T * 7 + E)
    ids, w = w4.moe_gate_topk(torch.from_numpy(logits).to(DEV), topk)
    w4.w4_device_status()
    o_ids, o_w = oracle.moe_gate_topk(logits, topk)
    assert np.array_equal(ids.cpu().numpy(), o_ids)                  # ids bit-exact
    assert np.allclose(w.cpu().numpy(), o_w, rtol=1e-5, atol=0)     # fp32 exp/sum order


def test_gate_topk_ties():
    """Integer logits: many exact ties, all broken toward the lower expert id."""
    rng = np.random.default_rng(5)
    logits = rng.integers(-3, 4, size=(300, 128)).astype(np.float32)
    ids, w = w4.moe_gate_topk(torch.from_numpy(logits).to(DEV), 8)
    o_ids, o_w = oracle.moe_gate_topk(logits, 8)
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    assert np.allclose(w.cpu().numpy(), o_w, rtol=1e-5, atol=0)


@pytest.mark.parametrize("S,F", [(1, 8), (3, 1536), (128, 1536), (2048, 1536), (7, 40)])
def test_silu_mul(S, F):
    gu = synth.normal_bf16((S, 2 * F), 2.0, seed=S + F)
    h = bits(w4.silu_mul(gu.to(DEV)))
    w4.w4_device_status()
    want = oracle.silu_mul(bits(gu))
    # FP32 silu on both sides; CUDA's expf and the host's exp may differ in the
    # last bit, which can move the BF16 rounding by one unit
    diff = np.abs(h.astype(np.int32) - want.astype(np.int32))
    assert diff.max() <= 1
    assert (diff == 0).mean() >= 0.999


@pytest.mark.parametrize("T,topk,N", [(1, 8, 8), (16, 8, 4096), (256, 8, 4096), (5, 3, 40)])
def test_combine(T, topk, N):
    D = synth.normal_bf16((T * topk, N), 1.0, seed=T + N)
    w = np.random.default_rng(T).random((T, topk)).astype(np.float32)
    out = bits(w4.moe_combine(D.to(DEV), torch.from_numpy(w).to(DEV)))
    w4.w4_device_status()
    assert np.array_equal(out, oracle.moe_combine(bits(D), w, topk))   # bit-exact


@pytest.mark.parametrize("T", [16, 64, 256])
def test_moe_layer_stage_by_stage(T):
    """One MoE decode layer on the GPU, each stage checked against the oracle fed
    the GPU's previous stage (so stage errors do not compound)."""
    cfg = synth.MoEDecode()
    E, topk, hidden, inter = cfg.E, cfg.topk, cfg.hidden, cfg.inter
    logits = _logits(T, E, seed=1000 + T)
    X = synth.normal_bf16((T, hidden), 1.0, seed=2000 + T)
    Wq_g, S_g, Wdq_g = _experts(E, 2 * inter, hidden)
    Wq_d, S_d, Wdq_d = _experts(E, hidden, inter)
    block = w4.w4_moe_block_size(T, topk, E)
    # gating
    ids, w = w4.moe_gate_topk(torch.from_numpy(logits).to(DEV), topk)
    o_ids, o_w = oracle.moe_gate_topk(logits, topk)
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    # align
    s_d, e_d, n_d = w4.moe_align(ids, E, block)
    s_o, e_o, n_o = oracle.moe_align(o_ids, E, block)
    assert int(n_d.item()) == n_o and np.array_equal(s_d.cpu().numpy(), s_o)
    # gate_up
    C1 = w4.moe_gemm(X.to(DEV), topk, torch.from_numpy(Wq_g).to(DEV), _np_bf16(S_g).to(DEV),
                     s_d, e_d, n_d, block, T * topk)
    _, R1 = oracle.moe_gemm(bits(X), topk, Wdq_g, s_o, e_o, n_o, T * topk, block)
    assert_gemm_close(bits(C1), R1, f"layer gate_up T={T}")
    # SiLU * up on the GPU's gate_up output
    H = w4.silu_mul(C1)
    diff = np.abs(bits(H).astype(np.int32) - oracle.silu_mul(bits(C1)).astype(np.int32))
    assert diff.max() <= 1
    # down on the GPU's h
    C2 = w4.moe_gemm(H, 1, torch.from_numpy(Wq_d).to(DEV), _np_bf16(S_d).to(DEV),
                     s_d, e_d, n_d, block, T * topk)
    _, R2 = oracle.moe_gemm(bits(H), 1, Wdq_d, s_o, e_o, n_o, T * topk, block)
    assert_gemm_close(bits(C2), R2, f"layer down T={T}")
    # combine of the GPU's down output with the GPU's weights
    out = w4.moe_combine(C2, w)
    w4.w4_device_status()
    assert np.array_equal(bits(out), oracle.moe_combine(bits(C2), w.cpu().numpy(), topk))


@pytest.mark.parametrize("T,E,N,K,block", [(16, 128, 4096, 1536, 16), (64, 128, 4096, 1536, 16),
                                            (256, 128, 4096, 1536, 32), (7, 8, 200, 256, 64),
                                            (33, 5, 136, 512, 16)])
def test_moe_down_combine_fused(T, E, N, K, block):
    """Down projection with the combine in its epilogue: C bit for bit the
    plain grouped GEMM's, out bit for bit w4_moe_combine / the oracle's combine
    of that C, twice on the same counters (left zero after each call)."""
    topk = 8 if E >= 8 else 3
    logits = _logits(T, E, seed=70 + T + N)
    ids, w = w4.moe_gate_topk(torch.from_numpy(logits).to(DEV), topk)
    H = synth.normal_bf16((T * topk, K), 1.0, seed=80 + T).to(DEV)
    Wq, S, _ = _experts(E, N, K)
    Wq_d, S_d = torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
    s_d, e_d, n_d = w4.moe_align(ids, E, block)
    cnt = torch.zeros(w4.w4_moe_combine_counter_bytes(T, N), dtype=torch.uint8, device=DEV)
    C_ref = bits(w4.moe_gemm(H, 1, Wq_d, S_d, s_d, e_d, n_d, block, T * topk))
    want = oracle.moe_combine(C_ref, w.cpu().numpy(), topk)
    for call in range(2):
        C, out = w4.moe_gemm_combine(H, Wq_d, S_d, s_d, e_d, n_d, block, w, cnt)
        w4.w4_device_status()
        assert np.array_equal(bits(C), C_ref), f"call {call}: C differs from the plain GEMM"
        assert np.array_equal(bits(out), want), f"call {call}: combine not bit-exact"
        assert int(cnt.count_nonzero()) == 0, f"call {call}: counters not reset"


def _silu_ref(R, F):
    """h = silu(g) * u from the oracle's FP32 gate_up sums (float64 evaluation)."""
    g, u = R[:, :F].astype(np.float64), R[:, F:].astype(np.float64)
    return (g / (1.0 + np.exp(-g)) * u).astype(np.float32)


@pytest.mark.parametrize("T,E,F,K,block", [(16, 128, 1536, 4096, 16), (64, 128, 1536, 4096, 64),
                                            (40, 8, 100, 1024, 16), (64, 8, 96, 512, 32)])
def test_moe_gate_up_silu_fused(T, E, F, K, block):
    """gate_up with SiLU*up in the epilogue against silu(g) * u of the oracle's FP32
    sums (the fused path never rounds g and u to BF16), and against the unfused
    chain (gate_up GEMM, then w4_silu_mul), which differs by that one rounding."""
    topk = 8
    logits = _logits(T, E, seed=50 + T + F)
    ids, w = w4.moe_gate_topk(torch.from_numpy(logits).to(DEV), topk)
    X = synth.normal_bf16((T, K), 1.0, seed=60 + T)
    Wq, S, Wdq = _experts(E, 2 * F, K)
    s_d, e_d, n_d = w4.moe_align(ids, E, block)
    canary = torch.full((T * topk, F), 0x7FC1, dtype=torch.int16).view(torch.bfloat16).to(DEV)
    Wq_d, S_d = torch.from_numpy(Wq).to(DEV), _np_bf16(S).to(DEV)
    H = w4.moe_gemm_silu(X.to(DEV), topk, Wq_d, S_d, s_d, e_d, n_d, block, T * topk, H=canary)
    w4.w4_device_status()
    Hb = bits(H)
    assert not np.any(Hb == 0x7FC1), "a real slot was left unwritten"
    o_ids, _ = oracle.moe_gate_topk(logits, topk)
    s_o, e_o, n_o = oracle.moe_align(o_ids, E, block)
    _, R = oracle.moe_gemm(bits(X), topk, Wdq, s_o, e_o, n_o, T * topk, block)
    assert_gemm_close(Hb, _silu_ref(R, F), f"fused silu T={T} F={F}")
    if F % 8 == 0:          # w4_silu_mul takes F in multiples of 8
        C1 = w4.moe_gemm(X.to(DEV), topk, Wq_d, S_d, s_d, e_d, n_d, block, T * topk)
        H2 = bits(w4.silu_mul(C1))
        assert_gemm_close(H2, _silu_ref(R, F), f"unfused silu T={T} F={F}")
