"""Host-side checks of the arithmetic the quantizer kernels use in place of
divisions (no GPU).  The fp32 fused operations are emulated exactly: every
product and sum below is exact in float64 for these operand sizes, and one
cast to float32 is the single rounding of the fused operation.

1. s32 = fl32(amax / 7) is formed as q0 = fl(a * c), r = fma(-q0, 7, a),
   q = fma(r, c, q0) with c = fl32(1/7) (quotient refinement with one FMA
   residual step, Markstein's method).  Checked for every finite BF16 amax.
2. The code rint_half_even(fl32(w / s)) is formed as
   fl(fl(fma(w, r, 1.5*2^13)) + (1.5*2^23 - 1.5*2^13)) with r an approximate
   reciprocal of s (relative error up to 2^-21 allowed): the FMA snaps w*r to
   the 2^-10 grid, which lands exact ties on the half-integer and leaves every
   other BF16/BF16 quotient (at least 1/510 from any half-integer) on its side;
   the add then rounds to an integer, ties to even.  Checked on every BF16
   magnitude below 128 group maxima, with the reciprocal perturbed both ways.
3. The zero-point quantizer's codes rint_half_even(fl32(x / s)), |x / s| < 3856,
   are formed the same way on the 2^-9 grid (snap constant 1.5*2^14).  Checked
   for every finite BF16 x in that range against every BF16 significand of s at
   three exponents (the subnormal edge, 1, 2^90), with every fp32 reciprocal
   within one ulp of 1/s and with a two-ulp perturbation both ways.
4. The NVFP4 quantizer's two band decisions: an FP32 quotient (group scale:
   amax * fl32(1 / fl32(6 g)); element: w * fl32(1 / fl32(E4M3(sc) * g)), the
   band folded into the reciprocal) is rounded at both ends of a relative band
   (2^-20, 2^-19); wherever the two ends agree, that code is the oracle's
   rounding of the FP64 quotient.  Checked for every BF16 value in range under
   several tensor scales; the FP32 arithmetic is numpy's IEEE float32.
"""
import numpy as np
import pytest

import oracle

F32 = np.float32
SNAP = 12288.0                 # 1.5 * 2^13
TOINT = 12582912.0 - 12288.0   # 1.5 * 2^23 - 1.5 * 2^13
MAGIC = 12582912.0             # 1.5 * 2^23


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def test_div7_refinement_exact_for_all_bf16():
    b = np.arange(0, 0x7F80, dtype=np.uint32)
    a = (b << 16).view(np.float32)
    ref = a / F32(7.0)
    c = float(F32(1.0) / F32(7.0))
    q0 = _f32(a.astype(np.float64) * c)
    r = _f32(a.astype(np.float64) - q0.astype(np.float64) * 7.0)
    q = _f32(r.astype(np.float64) * c + q0.astype(np.float64))
    assert np.array_equal(q.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("rel", [0.0, 2.0 ** -21, -(2.0 ** -21)])
def test_snap_rounding_matches_ieee_quotient(rel):
    all_bits = np.arange(0, 0x7F80, dtype=np.uint32)
    mags = (all_bits << 16).view(np.float32)
    for mant in range(0, 128, 3):
        amax = float(((np.uint32(0x4080 + mant)) << 16).view(np.float32))   # [4, 8)
        s_bits = oracle.bf16_from_f32_scalar(float(F32(amax) / F32(7.0)))
        s = float((np.uint32(s_bits) << 16).view(np.float32))
        w = mags[(mags <= amax)].astype(np.float64)
        w = np.concatenate([w, -w])
        ref = np.clip(np.rint((w.astype(np.float32) / F32(s)).astype(np.float64)), -8, 7)
        r = float(F32(1.0 / s)) * (1.0 + rel)
        a = _f32(w * r + SNAP)                       # fma(w, r, SNAP)
        c = _f32(a.astype(np.float64) + TOINT)       # fadd
        q = c.astype(np.float64) - MAGIC
        assert np.array_equal(q, ref), mant
        # the code is the low byte of the float's bits
        low = (c.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)
        assert np.array_equal(low.astype(np.float64), ref)


SNAP_Z = 24576.0                  # 1.5 * 2^14: ulp 2^-9 on [2^14, 2^15)
TOINT_Z = 12582912.0 - 24576.0    # 1.5 * 2^23 - 1.5 * 2^14


@pytest.mark.parametrize("s_exp", [-126, 0, 90])
def test_zero_point_snap_rounding_matches_ieee_quotient(s_exp):
    finite = np.arange(0, 0x7F80, dtype=np.uint32)
    mags = (finite << 16).view(np.float32).astype(np.float64)
    allx = np.concatenate([mags, -mags[1:]])
    for S in range(128, 256):
        s = S * 2.0 ** (s_exp - 7)                     # a normal BF16 scale
        x = allx[np.abs(allx) <= 3856.0 * s]
        ref = np.rint((x.astype(np.float32) / F32(s)).astype(np.float64))
        r0 = F32(1.0 / s)
        rs = [np.nextafter(r0, F32(0)), r0, np.nextafter(r0, F32(np.inf)),
              F32(float(r0) * (1.0 + 2.0 ** -22)), F32(float(r0) * (1.0 - 2.0 ** -22))]
        for r in rs:
            # fma(x, r, 1.5*2^14) lies in [2^14, 2^15): its one rounding puts
            # x*r (exact in float64) on the 2^-9 grid, ties to even
            k = np.rint(x * float(r) * 512.0)
            c = _f32(SNAP_Z + k / 512.0 + TOINT_Z)       # fadd: round to an integer
            q = c.astype(np.float64) - MAGIC
            assert np.array_equal(q, ref), (S, float(r))


_TENSOR_SCALES = [1.0, float(np.float32(2944.0) / np.float32(2688.0)),
                  float(np.float32(0.07) / np.float32(2688.0)), float(np.float32(3.1e-25))]


def _finite_positive_bf16():
    return (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("g", _TENSOR_SCALES)
def test_nvfp4_scale_band_decision(g):
    g32 = F32(g)
    enc = np.vectorize(oracle.e4m3_encode, otypes=[np.int64])
    amax = _finite_positive_bf16()
    amax = amax[amax.astype(np.float64) <= 2688.0 * float(g32) * (1 + 2.0 ** -20)]
    r6g = F32(1.0) / (F32(6.0) * g32)                    # fl32(1 / fl32(6 g))
    q = amax * r6g
    lo = enc((q * F32(1.0 - 2.0 ** -20)).astype(np.float64))
    hi = enc((q * F32(1.0 + 2.0 ** -20)).astype(np.float64))
    ref = enc(amax.astype(np.float64) / (6.0 * float(g32)))
    agree = lo == hi
    assert np.array_equal(lo[agree], ref[agree])
    assert (~agree).sum() <= max(200, len(amax) // 50)  # the FP64 path stays rare


@pytest.mark.parametrize("g", _TENSOR_SCALES)
def test_nvfp4_element_band_decision(g):
    g32 = F32(g)
    enc = np.vectorize(oracle.e2m1_encode, otypes=[np.int64])
    w_all = _finite_positive_bf16()
    w_all = np.concatenate([w_all, -w_all])
    for sc in (0x01, 0x07, 0x08, 0x2B, 0x38, 0x51, 0x7E):
        e = F32(oracle.e4m3_value(sc))
        step = float(e) * float(g32)                         # exact in FP64
        w = w_all[np.abs(w_all.astype(np.float64)) <= 7.0 * step]
        rs = F32(1.0) / (e * g32)                            # fl32(1 / fl32(E4M3(sc) g))
        lo = enc((w * (rs * F32(1.0 - 2.0 ** -19))).astype(np.float64)) & 7
        hi = enc((w * (rs * F32(1.0 + 2.0 ** -19))).astype(np.float64)) & 7
        ref = enc(w.astype(np.float64) / step) & 7            # magnitudes: the sign is w's
        agree = lo == hi
        assert agree.sum() > 0
        assert np.array_equal(lo[agree], ref[agree]), (sc, g)
        assert (~agree).sum() <= max(50, len(w) // 100)


def _bf16_rne(x64: np.ndarray) -> np.ndarray:
    """Round float64 values (exact results of a BF16 pair operation) to BF16,
    ties to even, as packed BF16 arithmetic does; returned as float64."""
    f = x64.astype(np.float32)          # exact here: the inputs below have <= 24 bits
    return oracle.bf16_to_f32(oracle.f32_to_bf16_bits(f)).astype(np.float64)


def test_zero_point_unpack_identity():
    """The zero-point unpack: OR-ing a nibble into BF16 128.0 gives 128 + q,
    subtracting 128 + z leaves q - z exactly, one multiply by the BF16 scale
    rounds (q - z) * s once, which is the oracle's dequantized value, for
    every code, every zero point and a spread of scales (normal, subnormal,
    large)."""
    q = np.arange(16)
    z = np.arange(16)
    qq, zz = np.meshgrid(q, z, indexing="ij")
    lhs_bits = (0x4300 | qq).astype(np.uint16)
    rhs_bits = (0x4300 | zz).astype(np.uint16)
    lhs = oracle.bf16_to_f32(lhs_bits).astype(np.float64)
    rhs = oracle.bf16_to_f32(rhs_bits).astype(np.float64)
    assert np.array_equal(lhs, 128.0 + qq) and np.array_equal(rhs, 128.0 + zz)
    diff = _bf16_rne(lhs - rhs)
    assert np.array_equal(diff, (qq - zz).astype(np.float64))
    rng = np.random.default_rng(1)
    s_bits = np.concatenate([rng.integers(0x0001, 0x7C00, 400), [0x0001, 0x0080, 0x3F80, 0x7C00]])
    for sb in s_bits.astype(np.uint16):
        s = float(oracle.bf16_to_f32(np.array([sb], np.uint16))[0])
        got = _bf16_rne(diff * s)
        # the oracle's value: bf16_rne of the exact product (q - z) * s
        want = np.array([[float(oracle.bf16_to_f32(np.array(
            [oracle.bf16_from_f32_scalar(float(np.float32((a - b) * s)))], np.uint16))[0])
            for b in z] for a in q])
        assert np.array_equal(got, want), hex(int(sb))
