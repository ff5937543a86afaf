"""The pins have teeth: plant one plausible mistake at a time in a temporary copy
of the oracle source (on the CPU, never in the committed oracle), rebuild it,
and check that at least one pin fails against the mutant."""
import os
import shutil

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "w4_oracle.c")

# (name, original text, mutated text, pins expected to catch it)
MUTANTS = [
    ("round_half_away", "float r = nearbyintf(y);", "float r = roundf(y);",
     [lambda: pins.test_hand_groups("group_A")]),
    ("round_truncate", "float r = nearbyintf(y);", "float r = truncf(y);",
     [lambda: pins.test_hand_groups("group_B")]),
    ("scale_qmax_8", "float s32 = amax / seven;", "float s32 = amax / (seven + 1.0f);",
     [lambda: pins.test_hand_groups("group_B"), pins.test_scale_exhaustive_exact]),
    ("scale_fp32_kept", "w4o_bf16_from_f32(s32);\n    float s = w4o_f32_from_bf16(s_bits);",
     "w4o_bf16_from_f32(s32);\n    float s = s32;",
     [lambda: pins.test_hand_groups("group_B")]),
    ("bf16_truncate", "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))",
     "if (0)", [lambda: pins.test_hand_groups("group_B")]),
    ("pack_high_first", "word |= ((uint32_t)q8[i] & 0xFu) << (4 * i);",
     "word |= ((uint32_t)q8[i] & 0xFu) << (4 * (7 - i));", [pins.test_pack_examples]),
    ("unpack_no_sign", "q8[i] = (int8_t)(v >= 8 ? v - 16 : v);", "q8[i] = (int8_t)v;",
     [pins.test_pack_examples]),
    ("amax_signed", "float a = fabsf(w4o_f32_from_bf16(w[i]));",
     "float a = w4o_f32_from_bf16(w[i]);", [lambda: pins.test_hand_groups("group_B")]),
    ("gemm_transposed_w", "w4o_f32_from_bf16(Wdq[n * K + k]);   /* exact */",
     "w4o_f32_from_bf16(Wdq[(k % N) * K + (n % K)]);",
     [lambda: pins.test_gemm_brute_force_fp64(3, 17, 96)]),
    ("gemm_dropped_term", "for (int64_t k = 0; k < K; ++k) {\n                float prod",
     "for (int64_t k = 1; k < K; ++k) {\n                float prod",
     [pins.test_gemm_one_hot_is_exact]),
    ("moe_align_descending", "for (int64_t i = 0; i < slots; ++i)       /* ascending slot order */",
     "for (int64_t i = slots - 1; i >= 0; --i)",
     [lambda: [pins.test_moe_align_brute_force(s) for s in range(40)]]),
    ("gate_ties_to_higher_id", "if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;",
     "if (!taken[e] && (best < 0 || l[e] >= l[best])) best = e;",
     [pins.test_moe_gate_topk_ties_go_to_lower_id]),
    ("gate_no_max_shift", "sum = sum + expf(l[e] - mx);", "sum = sum + expf(l[e]);",
     [lambda: pins.test_moe_gate_topk_brute_force(3, 8, 3, 1)]),
    ("combine_drops_last_k", "for (int64_t k = 0; k < topk; ++k) {\n                float prod = w[",
     "for (int64_t k = 0; k + 1 < topk; ++k) {\n                float prod = w[",
     [pins.test_moe_combine_reference_and_one_hot]),
    ("moe_align_no_pad", "total += (cnt[e] + block - 1) / block * block;", "total += cnt[e];",
     [lambda: [pins.test_moe_align_brute_force(s) for s in range(40)]]),
    ("zp_sign_flipped", "float zf = nearbyintf(0.0f - xmin / s);", "float zf = nearbyintf(xmin / s);",
     [lambda: pins.test_zp_exact_ramps(-5, 1)]),
    ("zp_dequant_adds_z", "float v = (float)((int)q - (int)z) * s;", "float v = (float)((int)q + (int)z) * s;",
     [lambda: pins.test_zp_exact_ramps(-5, 1)]),
    ("zp_no_upper_z_clamp", "if (zf > 15.0f) zf = 15.0f;", "",
     [pins.test_zp_brute_force_codes_and_zero_points]),
    ("zp_no_lower_z_clamp", "if (zf < 0.0f) zf = 0.0f;", "",
     [pins.test_zp_brute_force_codes_and_zero_points]),
    ("zp_range_is_max", "float range = xmax - xmin;", "float range = xmax;",
     [lambda: pins.test_zp_exact_ramps(-5, 1)]),
    ("zp_round_half_away", "float v = nearbyintf(y) + zf;", "float v = roundf(y) + zf;",
     [pins.test_zp_brute_force_codes_and_zero_points]),
    ("zp_pack_high_first", "word |= (uint32_t)(q8[i] & 0xFu) << (4 * i);",
     "word |= (uint32_t)(q8[i] & 0xFu) << (4 * (7 - i));",
     [pins.test_zp_pack_examples]),
    ("fp4_ties_up", "return (i % 2 == 0) ? i : i + 1;                 /* tie: the even code */",
     "return i + 1;", [pins.test_e2m1_table_and_rounding]),
    ("fp4_no_saturation", "if (a >= tab[n - 1]) return n - 1;", "if (a > 1e30) return n - 1;",
     [pins.test_e2m1_table_and_rounding]),
    ("mxfp4_exponent_off_by_one", "e = (ex - 1) - 2;                  /* floor(log2(amax)) - 2 */",
     "e = (ex - 1) - 1;", [pins.test_mxfp4_brute_force]),
    ("nvfp4_scale_over_7", "uint8_t sc = w4o_e4m3_encode(amax / (6.0 * (double)g));",
     "uint8_t sc = w4o_e4m3_encode(amax / (7.0 * (double)g));", [pins.test_nvfp4_brute_force]),
    ("e4m3_bias_8", "ldexp(1.0 + (double)m / 8.0, e - 7);", "ldexp(1.0 + (double)m / 8.0, e - 8);",
     [pins.test_e4m3_table_and_rounding]),
    # (random fp64 data has no exact ties, so the tie rule of this path is pinned
    # by group A through the INT4 path, not by the printed example)
    ("p4_scale_off_by_one", "double s = amax / (double)qmax;",
     "double s = amax / (double)(qmax + 1);", [pins.test_p4_int8_worked_example]),
    ("p4_amax_first_only", "if (fabs(x[g0 + i]) > amax) amax = fabs(x[g0 + i]);",
     "if (i == 0) amax = fabs(x[g0 + i]);", [pins.test_p4_int8_worked_example]),
]


@pytest.mark.parametrize("name,orig,mut,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, orig, mut, catchers, tmp_path, monkeypatch):
    text = open(SRC).read()
    assert text.count(orig) == 1, f"mutation site for {name} not unique"
    src = tmp_path / "w4_oracle_mutant.c"
    src.write_text(text.replace(orig, mut))
    so = str(tmp_path / "liboracle_mutant.so")
    oracle.compile_source(str(src), so)
    monkeypatch.setattr(oracle, "_lib", oracle.load_library(so))
    caught = False
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"no pin caught mutant {name}"


def test_unmutated_copy_passes(tmp_path, monkeypatch):
    src = tmp_path / "w4_oracle_copy.c"
    shutil.copy(SRC, src)
    so = str(tmp_path / "liboracle_copy.so")
    oracle.compile_source(str(src), so)
    monkeypatch.setattr(oracle, "_lib", oracle.load_library(so))
    pins.test_hand_groups("group_A")
    pins.test_hand_groups("group_B")
    pins.test_pack_examples()
    pins.test_gemm_one_hot_is_exact()
    pins.test_zp_exact_ramps(-5, 1)
    pins.test_zp_pack_examples()
