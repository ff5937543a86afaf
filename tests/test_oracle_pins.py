"""Pins of the CPU oracle against what the sources and the mathematics fix.

No GPU.  Each test checks the oracle against something other than itself: a
worked example printed on a page, a hand-worked group, exact rational
arithmetic, an exhaustive enumeration, a closed-form bound, or brute force on
tiny inputs.
"""
import json
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests._exact import (bf16_bits_to_fraction, fraction_to_bf16_bits,
                          round_half_even)

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _bf16_bits(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _u32(x):
    return int(x) & 0xFFFFFFFF


# ---------------------------------------------------------------------------
# Worked example printed on the quantization-basics page (§6.1)
# ---------------------------------------------------------------------------

def test_p4_int8_worked_example():
    g = _load("p4_int8_worked_example.json")
    rng = np.random.default_rng(42)
    w = rng.standard_normal(200_000) * 0.05
    w[:500] *= 6.0
    w16 = w.astype(np.float16).astype(np.float64)
    q, s = oracle.symmetric_quantize_f64(w16, qmax=127)
    s = float(s[0])
    err = q.astype(np.float64) * s - w16
    p = g["printed"]
    assert f"{s:.6f}" == p["scale_s"]
    assert f"{s / 2:.6f}" == p["half_scale"]
    assert f"{np.abs(err).max():.6f}" == p["max_abs_err"]
    assert f"{np.abs(err).mean():.6f}" == p["mae"]
    assert f"{100 * np.linalg.norm(err) / np.linalg.norm(w16):.6f}" == p["rel_l2_percent"]
    assert len(np.unique(q)) == p["distinct_codes"]


# ---------------------------------------------------------------------------
# Hand-worked INT4 groups
# ---------------------------------------------------------------------------

def _group_b_bits():
    vals = (torch.arange(32, dtype=torch.float32) - 16) * torch.tensor(0.001, dtype=torch.float32)
    return vals.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["group_A", "group_B"])
def test_hand_groups(name):
    g = _load("hand_groups.json")[name]
    W = (_bf16_bits(g["inputs"]) if "inputs" in g else _group_b_bits()).reshape(1, 32)
    q, S = oracle.quantize(W)
    assert int(S[0, 0]) == int(g["scale_bits"], 16)
    assert q[0].tolist() == g["q"]
    Wq, S2 = oracle.quantize_pack(W)
    assert [_u32(x) for x in Wq[0]] == [int(h, 16) for h in g["words"]]
    assert int(S2[0, 0]) == int(g["scale_bits"], 16)
    # fake quant and dequant-of-export give bf16(q * s) -- checked in exact arithmetic
    Wdq, S3 = oracle.fake_quant(W)
    s = bf16_bits_to_fraction(int(g["scale_bits"], 16))
    want = [fraction_to_bf16_bits(Fraction(qi) * s) for qi in g["q"]]
    assert [int(b) for b in Wdq[0]] == want
    assert [int(b) for b in oracle.dequant(Wq, S2)[0]] == want
    if name == "group_B":
        w = [bf16_bits_to_fraction(int(b)) for b in W[0]]
        assert max(w, key=abs) == Fraction(g["amax"]) * (-1)
        errs = [abs(wi - qi * s) for wi, qi in zip(w, g["q"])]
        assert max(errs) == Fraction(g["max_abs_err_exact"])
        assert max(errs) <= s / 2 == Fraction(g["half_scale"])


def test_pack_examples():
    g = _load("hand_groups.json")
    for key in ("pack_C", "pack_D"):
        q = np.array(g[key]["q"], np.int8)
        word = oracle.pack(q)[0]
        assert _u32(word) == int(g[key]["word"], 16)
        assert int(word) == g[key]["int32"]
        assert oracle.unpack(np.array([word], np.int32)).tolist() == g[key]["q"]


# ---------------------------------------------------------------------------
# Packing: exhaustive over value x position, and round trips
# ---------------------------------------------------------------------------

def test_pack_exhaustive_value_position():
    for pos in range(8):
        for v in range(-8, 8):
            q = np.zeros(8, np.int8)
            q[pos] = v
            word = _u32(oracle.pack(q)[0])
            assert word == ((v & 0xF) << (4 * pos)), (pos, v)
            assert oracle.unpack(np.array([np.int32(np.uint32(word).view(np.int32))])).tolist() == q.tolist()


def test_pack_round_trips():
    rng = np.random.default_rng(7)
    words = rng.integers(-2**31, 2**31, size=1 << 20, dtype=np.int64).astype(np.int32)
    words[:4] = np.array([0, -1, 0x7FFFFFFF, -2004318072], np.int64).astype(np.int32)
    q = oracle.unpack(words)
    assert q.min() >= -8 and q.max() <= 7
    assert np.array_equal(oracle.pack(q), words)
    codes = rng.integers(-8, 8, size=(1 << 16, 8)).astype(np.int8)
    assert np.array_equal(oracle.unpack(oracle.pack(codes)), codes)


# ---------------------------------------------------------------------------
# Scale: exhaustive over every positive finite BF16 amax, in exact arithmetic
# ---------------------------------------------------------------------------

def test_scale_exhaustive_exact():
    amax_bits = np.arange(1, 0x7F80, dtype=np.uint16)          # all positive finite
    W = np.zeros((amax_bits.size, 32), np.uint16)
    W[:, 0] = amax_bits
    W[:, 1] = amax_bits | 0x8000                                 # a negative twin
    _, S = oracle.quantize(W)
    got = S[:, 0]
    for i, b in enumerate(amax_bits.tolist()):
        want = fraction_to_bf16_bits(bf16_bits_to_fraction(b) / 7)
        assert int(got[i]) == want, hex(b)


# ---------------------------------------------------------------------------
# Codes: the rounding decision against exact rational arithmetic
# ---------------------------------------------------------------------------

def _structured_groups():
    """Groups whose amax sweeps all 128 BF16 mantissas of [4, 8) and whose other
    31 entries sweep every BF16 magnitude below amax (both signs)."""
    rows = []
    all_bits = np.arange(0, 0x7F80, dtype=np.uint16)
    mags = bf16_f = (all_bits.astype(np.uint32) << 16).view(np.float32)
    for mant in range(128):
        amax_bits = np.uint16(0x4080 + mant)                    # [4, 8)
        amax = float((np.uint32(amax_bits) << 16).view(np.float32))
        cand = all_bits[(mags <= amax) & (mags >= amax * 2.0 ** -12)]
        cand = np.concatenate([cand, cand | np.uint16(0x8000)])
        for c0 in range(0, cand.size, 31):
            chunk = cand[c0:c0 + 31]
            row = np.zeros(32, np.uint16)
            row[0] = amax_bits
            row[1:1 + chunk.size] = chunk
            rows.append(row)
    return np.stack(rows)


def test_codes_match_exact_rounding():
    W = _structured_groups()
    q, S = oracle.quantize(W)
    # full set: the float64 quotient lies within 2**-52 of w/s while a non-tie
    # w/s (both BF16) is at least 1/510 from any half-integer, so rounding the
    # float64 quotient half-to-even gives the exact decision.
    w = (W.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = (S[:, :1].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = np.clip(np.rint(w / s), -8, 7).astype(np.int8)
    assert np.array_equal(q, want)
    # a random sample in exact rational arithmetic
    rnd = random.Random(3)
    for _ in range(3000):
        r = rnd.randrange(W.shape[0])
        c = rnd.randrange(32)
        wf = bf16_bits_to_fraction(int(W[r, c]))
        sf = bf16_bits_to_fraction(int(S[r, 0]))
        assert int(q[r, c]) == max(-8, min(7, round_half_even(wf / sf)))


def test_clamp_never_fires_and_code_minus8_unused():
    for seed in range(4):
        W = torch.randn(256, 1024, generator=torch.Generator().manual_seed(seed))
        W[W.abs() > 2] *= 20
        bits = W.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        q, _ = oracle.quantize(bits)
        assert q.min() >= -7 and q.max() <= 7


# ---------------------------------------------------------------------------
# Error bound |w - q s| <= s/2 (quantization-basics page, §2.4)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dist", ["normal_outliers", "laplace"])
def test_error_bound(dist):
    import synth
    if dist == "normal_outliers":
        W = synth.normal_bf16((384, 2048), 0.02, seed=11, outlier_frac=0.001)
    else:
        W = synth.laplace_bf16((384, 2048), 0.015, seed=12)
    bits = synth.bits(W)
    q, S = oracle.quantize(bits)
    w = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = np.repeat((S.astype(np.uint32) << 16).view(np.float32).astype(np.float64), 32, axis=1)
    assert np.all(np.abs(w - q * s) <= s / 2 * (1 + 2.0 ** -20))
    # the BF16 dequantized value adds at most half an ulp of itself
    Wdq, _ = oracle.fake_quant(bits)
    d = (Wdq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = np.where(d == 0, 0.0, 2.0 ** (np.floor(np.log2(np.abs(np.where(d == 0, 1, d)))) - 7))
    assert np.all(np.abs(w - d) <= s / 2 + ulp / 2)
    # mean absolute error ~ s/4 under uniform rounding error (§6.1 remark): soft check
    ratio = np.mean(np.abs(w - q * s)) / np.mean(s)
    assert 0.2 < ratio < 0.3


def test_zero_group_and_tiny_group():
    W = np.zeros((2, 64), np.uint16)
    W[1, 32] = 0x0001                      # smallest subnormal: amax/7 rounds to 0
    W[1, 33] = 0x8001
    q, S = oracle.quantize(W)
    assert np.all(S == 0) and np.all(q == 0)
    Wdq, _ = oracle.fake_quant(W)
    assert np.all(Wdq == 0)                # +0.0, not -0.0


def test_fake_quant_equals_dequant_of_export():
    import synth
    bits = synth.bits(synth.normal_bf16((512, 1024), 0.02, seed=21, outlier_frac=0.001))
    Wdq, S = oracle.fake_quant(bits)
    Wq, S2 = oracle.quantize_pack(bits)
    assert np.array_equal(S, S2)
    assert np.array_equal(Wdq, oracle.dequant(Wq, S2))


def test_ste_is_identity():
    rng = np.random.default_rng(0)
    g = rng.integers(0, 1 << 16, size=4096, dtype=np.uint32).astype(np.uint16)
    assert np.array_equal(oracle.ste_backward(g), g)


# ---------------------------------------------------------------------------
# GEMM: brute force in fp64 on tiny shapes, one-hot exactness
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (3, 17, 96), (8, 64, 256), (5, 40, 160)])
def test_gemm_brute_force_fp64(M, N, K):
    import synth
    W = synth.bits(synth.normal_bf16((N, K), 0.02, seed=M * 100 + N))
    X = synth.bits(synth.normal_bf16((M, K), 1.0, seed=M * 100 + N + 1))
    Wdq, _ = oracle.fake_quant(W)
    Y, R = oracle.gemm(X, Wdq)
    x = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = (Wdq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = np.zeros((M, N))
    for m in range(M):                      # plain triple loop in fp64
        for n in range(N):
            exact[m, n] = sum(x[m, k] * w[n, k] for k in range(K))
    bound = K * 2.0 ** -24 * (np.abs(x) @ np.abs(w).T)
    assert np.all(np.abs(R - exact) <= bound)
    assert np.allclose(exact, x @ w.T, rtol=0, atol=1e-12)   # library cross-check
    y = (Y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(y - R) <= np.abs(R) * 2.0 ** -8)
    # the packed-input GEMM is the same product
    Wq, S = oracle.quantize_pack(W)
    Y2, R2 = oracle.w4a16_gemm(X, Wq, S)
    assert np.array_equal(Y2, Y) and np.array_equal(R2, R)


def test_gemm_one_hot_is_exact():
    import synth
    N, K = 48, 128
    W = synth.bits(synth.normal_bf16((N, K), 0.02, seed=5, outlier_frac=0.01))
    Wdq, _ = oracle.fake_quant(W)
    X = np.zeros((K, K), np.uint16)
    X[np.arange(K), np.arange(K)] = 0x3F80        # 1.0
    Y, R = oracle.gemm(X, Wdq)
    assert np.array_equal(Y, Wdq.T)


# ---------------------------------------------------------------------------
# moe_align: brute force on tiny inputs and invariants
# ---------------------------------------------------------------------------

def _brute_moe_align(ids, E, block):
    T, topk = ids.shape
    slots = T * topk
    flat = ids.reshape(-1).tolist()
    out, experts = [], []
    for e in range(E):
        mine = [i for i in range(slots) if flat[i] == e]
        if not mine:
            continue
        padded = -(-len(mine) // block) * block
        out += mine + [slots] * (padded - len(mine))
        experts += [e] * (padded // block)
    return out, experts


@pytest.mark.parametrize("seed", range(40))
def test_moe_align_brute_force(seed):
    rnd = random.Random(seed)
    T = rnd.choice([1, 2, 3, 5, 9])
    topk = rnd.choice([1, 2, 4])
    E = rnd.choice([1, 3, 8, 16])
    block = rnd.choice([1, 2, 4, 16])
    ids = np.array([[rnd.randrange(E) for _ in range(topk)] for _ in range(T)], np.int32)
    sorted_ids, expert_ids, npp = oracle.moe_align(ids, E, block)
    want, want_e = _brute_moe_align(ids, E, block)
    assert npp == len(want)
    assert sorted_ids[:npp].tolist() == want
    assert np.all(sorted_ids[npp:] == T * topk)
    assert expert_ids[:npp // block].tolist() == want_e
    assert np.all(expert_ids[npp // block:] == -1)
    real = sorted_ids[sorted_ids < T * topk]
    assert sorted(real.tolist()) == list(range(T * topk))       # each slot once


def test_moe_align_skips_out_of_range_ids():
    ids = np.array([[0, 5], [-1, 1]], np.int32)
    sorted_ids, expert_ids, npp = oracle.moe_align(ids, E=2, block=2)
    assert sorted_ids[:npp].tolist() == [0, 4, 3, 4]
    assert expert_ids[:2].tolist() == [0, 1]


def test_moe_gemm_equals_dense_rows():
    import synth
    E, N, K, T, topk, block = 4, 24, 64, 5, 2, 4
    ids, _ = synth.routing(T, E, topk, seed=9)
    A = synth.bits(synth.normal_bf16((T, K), 1.0, seed=10))
    W = synth.bits(synth.normal_bf16((E, N, K), 0.02, seed=11))
    Wdq = np.stack([oracle.fake_quant(W[e])[0] for e in range(E)])
    sorted_ids, expert_ids, npp = oracle.moe_align(ids.numpy(), E, block)
    canary = np.full((T * topk, N), 0x7FC1, np.uint16)
    C, R = oracle.moe_gemm(A, topk, Wdq, sorted_ids, expert_ids, npp, T * topk, block,
                           C_init=canary)
    flat = ids.numpy().reshape(-1)
    for slot in range(T * topk):
        Yd, Rd = oracle.gemm(A[slot // topk:slot // topk + 1], Wdq[flat[slot]])
        assert np.array_equal(C[slot], Yd[0]) and np.array_equal(R[slot], Rd[0])


# ---------------------------------------------------------------------------
# MoE layer glue: gating, SiLU-gated product, weighted combine
# ---------------------------------------------------------------------------

def _brute_gate(logits, topk):
    """Independent restatement: sort experts by (-logit, id) with Python's sort,
    probabilities from a float64 softmax."""
    ids, ws = [], []
    for row in logits.astype(np.float64):
        order = sorted(range(len(row)), key=lambda e: (-row[e], e))[:topk]
        p = np.exp(row - row.max())
        p /= p.sum()
        ids.append(order)
        ws.append([p[e] for e in order])
    return np.array(ids, np.int32), np.array(ws)


@pytest.mark.parametrize("T,E,topk,seed", [(1, 1, 1, 0), (3, 8, 3, 1), (17, 128, 8, 2),
                                           (5, 33, 33, 3), (9, 256, 32, 4)])
def test_moe_gate_topk_brute_force(T, E, topk, seed):
    logits = np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.moe_gate_topk(logits, topk)
    want_ids, want_w = _brute_gate(logits, topk)
    assert np.array_equal(ids, want_ids)
    assert np.allclose(w, want_w, rtol=2e-6, atol=0)
    assert np.all(np.diff(w, axis=1) <= 0)                  # descending
    if topk == E:
        assert np.allclose(w.sum(axis=1), 1.0, rtol=1e-5)    # all of the softmax


def test_moe_gate_topk_ties_go_to_lower_id():
    logits = np.array([[1.0, 3.0, 3.0, -2.0, 3.0, 0.5],
                       [0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], np.float32)
    ids, w = oracle.moe_gate_topk(logits, 4)
    assert ids.tolist() == [[1, 2, 4, 0], [0, 1, 2, 3]]
    assert np.allclose(w[1], 1.0 / 6.0, rtol=1e-6)
    assert w[0, 0] == w[0, 1] == w[0, 2]


def test_moe_gate_topk_shift_invariant():
    """softmax(l + c) = softmax(l): the same ids, weights within fp32 rounding."""
    logits = np.random.default_rng(7).standard_normal((6, 64)).astype(np.float32)
    a_ids, a_w = oracle.moe_gate_topk(logits, 8)
    b_ids, b_w = oracle.moe_gate_topk(logits + np.float32(40.0), 8)
    assert np.array_equal(a_ids, b_ids)
    assert np.allclose(a_w, b_w, rtol=1e-5)


def test_moe_combine_reference_and_one_hot():
    rng = np.random.default_rng(3)
    T, topk, N = 7, 4, 24
    D = oracle.f32_to_bf16_bits(rng.standard_normal((T * topk, N)).astype(np.float32))
    w = rng.random((T, topk)).astype(np.float32)
    out = oracle.moe_combine(D, w, topk)
    Df = oracle.bf16_to_f32(D).astype(np.float64).reshape(T, topk, N)
    ref = np.einsum("tk,tkn->tn", w.astype(np.float64), Df)
    got = oracle.bf16_to_f32(out).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)   # BF16 rounding
    # one-hot weights pick a slot row exactly
    w1 = np.zeros((T, topk), np.float32)
    w1[np.arange(T), np.arange(T) % topk] = 1.0
    out1 = oracle.moe_combine(D, w1, topk)
    assert np.array_equal(out1, D.reshape(T, topk, N)[np.arange(T), np.arange(T) % topk])


def test_silu_mul_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 30.0, -30.0, 2.0], np.float32)
    u = np.array([5.0, 2.0, 2.0, 1.0, 1.0, 0.0], np.float32)
    gu = oracle.f32_to_bf16_bits(np.concatenate([g, u])[None, :])
    h = oracle.bf16_to_f32(oracle.silu_mul(gu))[0].astype(np.float64)
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    want = gd / (1.0 + np.exp(-gd)) * ud          # silu(g) * u in float64
    assert h[0] == 0.0 and h[5] == 0.0            # silu(0) = 0; u = 0
    assert h[3] == 30.0                           # silu(x) -> x for large x
    assert abs(h[4]) < 1e-11                      # silu(x) -> 0 for very negative x
    assert np.all(np.abs(h - want) <= 2.0 ** -8 * np.abs(want))   # one BF16 rounding


# ---------------------------------------------------------------------------
# Asymmetric (zero-point) groups: the affine map of the quantization tutorial
# (§2.1) with the asymmetric scale and zero point of its §2.3, unsigned INT4
# codes [0, 15].  Pinned by exact ramps, by brute force over the 16 codes in
# exact rational arithmetic, and by the tutorial's |x^ - x| <= s/2 bound (§2.4).
# ---------------------------------------------------------------------------

def _zp_group(values, exact=True):
    bits = np.array([fraction_to_bf16_bits(Fraction(v)) for v in values], np.uint16)
    if exact:
        assert [bf16_bits_to_fraction(int(b)) for b in bits] == [Fraction(v) for v in values]
    return bits.reshape(1, -1)


@pytest.mark.parametrize("lo,step", [(0, 1), (-5, 1), (-15, 1), (-7, Fraction(1, 64)),
                                     (-3, 4), (0, Fraction(3, 8))])
def test_zp_exact_ramps(lo, step):
    # values lo*step ... (lo+15)*step, twice: x_max - x_min = 15 step, so s = step,
    # z = -lo, every code q = i and x^ = x exactly
    vals = [Fraction(lo + i) * step for i in range(16)] * 2
    q, S, Z = oracle.quantize_zp(_zp_group(vals))
    assert bf16_bits_to_fraction(int(S[0, 0])) == Fraction(step)
    assert int(Z[0, 0]) == -lo
    assert q[0].tolist() == list(range(16)) * 2
    Wq, S2, Z2 = oracle.quantize_pack_zp(_zp_group(vals))
    back = [bf16_bits_to_fraction(int(b)) for b in oracle.dequant_zp(Wq, S2, Z2)[0]]
    assert back == vals


def _brute_zp(vals, s, z):
    """Codes by brute force: the nearest of (c - z) * s, c in [0, 15], to each x,
    ties to the even c - z; exact rationals."""
    out = []
    for x in vals:
        best = None
        for c in range(16):
            d = abs(x - (c - z) * s)
            key = (d, (c - z) % 2)
            if best is None or key < best[0]:
                best = (key, c)
        out.append(best[1])
    return out


def test_zp_brute_force_codes_and_zero_points():
    rng = random.Random(7)
    for trial in range(300):
        kind = trial % 5
        if kind == 0:      # straddles zero
            vals = [Fraction(rng.randint(-200, 200), 64) for _ in range(32)]
        elif kind == 1:    # all positive: z clamps at 0, top codes clamp at 15
            vals = [Fraction(rng.randint(40, 300), 32) for _ in range(32)]
        elif kind == 2:    # all negative: z clamps at 15
            vals = [Fraction(-rng.randint(40, 300), 32) for _ in range(32)]
        elif kind == 3:    # wide dynamic range
            vals = [Fraction(rng.choice([-1, 1]) * rng.randint(1, 255), 2 ** rng.randint(0, 12))
                    for _ in range(32)]
        else:              # few distinct values, many ties
            vals = [Fraction(rng.randint(-8, 8), 4) for _ in range(32)]
        bits = _zp_group(vals, exact=False)     # rounded to BF16, then read back
        vals = [bf16_bits_to_fraction(int(b)) for b in bits[0]]
        q, S, Z = oracle.quantize_zp(bits)
        s = bf16_bits_to_fraction(int(S[0, 0]))
        rng_x = max(vals) - min(vals)
        if rng_x == 0:
            assert s == 0 and int(Z[0, 0]) == 0 and q.max() == 0
            continue
        # s is the BF16 nearest (within half a BF16 ulp, plus the fp32 step) to range / 15
        assert abs(s - rng_x / 15) <= s / 256 + s / 2 ** 20, (trial, s, rng_x)
        # z: the integer in [0, 15] nearest to -x_min / s, ties to even
        zt = -min(vals) / s
        zc = min(range(16), key=lambda c: (abs(c - zt), c % 2))
        assert int(Z[0, 0]) == zc, (trial, zt)
        assert q[0].tolist() == _brute_zp(vals, s, zc), trial
        # the group's minimum maps to code 0 whenever z is not clamped
        if 0 <= round_half_even(zt) <= 15:
            assert q[0][vals.index(min(vals))] == 0


def test_zp_error_bound_half_step():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 256)) * 0.05 + rng.uniform(-0.05, 0.05, (64, 1))).astype(np.float32)
    W = oracle.f32_to_bf16_bits(x)
    Wq, S, Z = oracle.quantize_pack_zp(W)
    back = oracle.bf16_to_f32(oracle.dequant_zp(Wq, S, Z)).astype(np.float64)
    xv = oracle.bf16_to_f32(W).astype(np.float64)
    s = np.repeat(oracle.bf16_to_f32(S).astype(np.float64), 32, axis=1)
    z = np.repeat(Z.astype(np.int64), 32, axis=1)
    unclamped = (np.rint(xv / s) + z >= 0) & (np.rint(xv / s) + z <= 15)
    assert unclamped.mean() > 0.99
    # |x^ - x| <= s / 2, plus the BF16 rounding of (q - z) * s (half an ulp, 2^-8 relative)
    err = np.abs(back - xv)
    assert np.all(err[unclamped] <= s[unclamped] / 2 + np.abs(back[unclamped]) * 2.0 ** -8 + 1e-30)


def test_zp_pack_examples():
    assert oracle.pack_u(np.arange(8, dtype=np.uint8))[0] == 0x76543210
    w = oracle.pack_u(np.arange(8, 16, dtype=np.uint8))[0]
    assert (int(w) & 0xFFFFFFFF) == 0xFEDCBA98
    words = np.array([0x76543210, np.int32(-0x01234568)], np.int32)     # 0xFEDCBA98
    assert oracle.unpack_u(words).tolist() == list(range(16))


# ---------------------------------------------------------------------------
# Micro-scaled FP4 (the MR-GPTQ / QuTLASS summary page: MXFP4 with one scale
# per 32 elements, NVFP4 with one per 16).  The element and scale formats are
# decoded here from their bit-field definitions (sign, exponent with bias,
# mantissa), independently of the oracle's tables; codes are checked by brute
# force over every code in exact rationals.
# ---------------------------------------------------------------------------

def _minifloat(code: int, ebits: int, mbits: int, bias: int) -> Fraction:
    sign = -1 if code >> (ebits + mbits) & 1 else 1
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    if e == 0:
        return sign * Fraction(m, 1 << mbits) * Fraction(2) ** (1 - bias)
    return sign * (1 + Fraction(m, 1 << mbits)) * Fraction(2) ** (e - bias)


def _e2m1(c):
    return _minifloat(c, 2, 1, 1)


def _e4m3(c):
    return _minifloat(c, 4, 3, 7)


def _nearest_code(x: Fraction, codes, value):
    """Nearest representable value to x among codes, ties to the even code; a
    zero result takes the positive code."""
    best = None
    for c in codes:
        key = (abs(x - value(c)), c & 1, c)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_e2m1_table_and_rounding():
    for c in range(16):
        assert Fraction(oracle.e2m1_value(c)) == _e2m1(c)
    assert [float(_e2m1(c)) for c in range(8)] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    rng = random.Random(3)
    pts = [Fraction(k, 8) for k in range(-64, 65)] + [Fraction(rng.randint(-900, 900), 97) for _ in range(300)]
    for x in pts:
        want = _nearest_code(x, [c for c in range(16) if c != 8], _e2m1)
        assert oracle.e2m1_encode(float(x)) == want, x
    # midpoints go to the even code; magnitudes above 6 saturate
    assert [oracle.e2m1_encode(v) for v in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0)] == \
        [0, 2, 2, 4, 4, 6, 6, 7, 7]


def test_e4m3_table_and_rounding():
    for c in range(127):
        assert Fraction(oracle.e4m3_value(c)) == _e4m3(c), c
    assert oracle.e4m3_value(126) == 448.0 and oracle.e4m3_value(1) == 2.0 ** -9
    rng = random.Random(5)
    for _ in range(2000):
        x = Fraction(rng.randint(1, 1 << 20), 1 << rng.randint(0, 40))
        want = _nearest_code(x, range(127), _e4m3)
        assert oracle.e4m3_encode(float(x)) == want, x
    assert oracle.e4m3_encode(1000.0) == 126             # saturates at 448
    assert oracle.e4m3_encode(2.0 ** -11) == 0            # below half the smallest step: 0


def test_mxfp4_brute_force():
    rng = random.Random(13)
    for trial in range(120):
        scale = Fraction(2) ** rng.randint(-20, 10)
        vals = [scale * Fraction(rng.randint(-4000, 4000), 512) for _ in range(32)]
        if trial % 10 == 0:
            vals = [Fraction(0)] * 32
        bits = np.array([fraction_to_bf16_bits(v) for v in vals], np.uint16).reshape(1, -1)
        xs = [bf16_bits_to_fraction(int(b)) for b in bits[0]]
        q, E = oracle.quantize_mxfp4(bits)
        amax = max(abs(x) for x in xs)
        if amax == 0:
            assert int(E[0, 0]) == 127 and q.max() == 0
            continue
        e = 0
        while Fraction(2) ** e > amax:
            e -= 1
        while Fraction(2) ** (e + 1) <= amax:
            e += 1
        assert int(E[0, 0]) == e - 2 + 127, trial
        X = Fraction(2) ** (e - 2)
        for i, x in enumerate(xs):
            want = _nearest_code(x / X, [c for c in range(16) if c != 8], _e2m1)
            assert int(q[0, i]) == want, (trial, i)
        # dequant: value * 2^e, exact, then BF16
        back = oracle.dequant_mxfp4(q, E)[0]
        assert [bf16_bits_to_fraction(int(b)) for b in back] == \
            [bf16_bits_to_fraction(fraction_to_bf16_bits(_e2m1(int(c)) * X)) for c in q[0]]


def test_nvfp4_brute_force():
    rng = np.random.default_rng(17)
    x = (rng.standard_normal((6, 64)) * np.exp(rng.uniform(-3, 3, (6, 4))).repeat(16, axis=1)).astype(np.float32)
    W = oracle.f32_to_bf16_bits(x)
    q, S, g = oracle.quantize_nvfp4(W)
    xs = [[bf16_bits_to_fraction(int(b)) for b in row] for row in W]
    amax_t = max(abs(v) for row in xs for v in row)
    assert np.float32(g) == np.float32(np.float32(float(amax_t)) / np.float32(2688.0))
    gF = Fraction(float(np.float32(g)))
    for r in range(W.shape[0]):
        for j in range(W.shape[1] // 16):
            grp = xs[r][16 * j:16 * j + 16]
            amax = max(abs(v) for v in grp)
            sc = _nearest_code(amax / (6 * gF), range(127), _e4m3)
            assert int(S[r, j]) == sc, (r, j)
            step = _e4m3(sc) * gF
            for i, v in enumerate(grp):
                want = 0 if step == 0 else _nearest_code(v / step, [c for c in range(16) if c != 8], _e2m1)
                assert int(q[r, 16 * j + i]) == want, (r, j, i)
