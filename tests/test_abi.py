"""The C-ABI library loads, exports every entry point include/w4a16.h declares,
and rejects malformed calls on the host before launching anything (no GPU)."""
import ctypes
import os
import re

import pytest

import int4_w4a16_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4\w*)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["w4_fake_quant", "w4_ste_backward", "w4_quantize_pack", "w4_dequant",
                     "w4a16_gemm", "w4a16_gemm_workspace_bytes", "w4_moe_align",
                     "w4_moe_w4a16_gemm", "w4_moe_capacity", "w4_moe_gate_topk",
                     "w4_moe_block_size", "w4_silu_mul", "w4_moe_combine", "w4_qat_gemm",
                     "w4_moe_w4a16_gemm_silu", "w4_quantize_pack_zp", "w4_dequant_zp",
                     "w4a16_gemm_zp",
                     "w4_device_status", "w4_status_string", "w4_version",
                     "w4_last_cuda_error"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(w4.LIB_PATH)
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in w4a16.h but not exported"


def test_status_strings_and_version():
    L = w4.lib()
    assert [L.w4_status_string(i) for i in range(5)] == [
        b"W4_OK", b"W4_ERR_INVALID_ARG", b"W4_ERR_UNSUPPORTED", b"W4_ERR_CUDA",
        b"W4_ERR_TIMEOUT"]
    assert w4.w4_version() >= 100


def test_moe_capacity_host_only():
    L = w4.lib()
    assert L.w4_moe_capacity(16, 8, 128, 16) == 16 * 8 + 128 * 15
    assert L.w4_moe_capacity(3, 2, 4, 4) == 20          # 6 + 12 = 18 -> 20
    assert L.w4_moe_capacity(-1, 8, 128, 16) == 0


A16 = 0x10000          # a 16-byte-aligned fake address: never dereferenced, the
MIS = 0x10002          # calls below all fail validation before any CUDA call


@pytest.mark.parametrize("args,expect", [
    ((A16, A16, None, 4, 64, 16, None), 2),      # group != 32 -> unsupported
    ((A16, A16, None, 4, 48, 32, None), 1),      # K not a multiple of 32
    ((None, A16, None, 4, 64, 32, None), 1),     # null input
    ((MIS, A16, None, 4, 64, 32, None), 1),      # misaligned input
    ((A16, A16, None, 4, 64, 32, None), 1),      # output aliases input
    ((A16, A16 + 0x1000, MIS, 4, 64, 32, None), 1),  # misaligned scales
    ((A16, A16 + 0x1000, None, -1, 64, 32, None), 1),  # negative rows
])
def test_fake_quant_validation(args, expect):
    assert w4.lib().w4_fake_quant(*args) == expect


def test_other_validation():
    L = w4.lib()
    assert L.w4_quantize_pack(A16, A16 + 0x100, None, 4, 64, 32, None) == 1
    assert L.w4_quantize_pack(A16, A16 + 0x100, A16 + 0x200, 4, 64, 8, None) == 2
    assert L.w4_dequant(A16, MIS, A16 + 0x100, 4, 64, 32, None) == 1
    assert L.w4_ste_backward(A16, MIS, 8, None) == 1
    assert L.w4_wait_selftest(0, None) == 1                    # limit out of range
    assert L.w4_wait_selftest(2000000, None) == 1
    assert L.w4_ste_backward(A16, A16, 8, None) == 0           # aliased: zero-copy no-op
    assert L.w4_ste_backward(A16, A16 + 2 * 8, 64, None) == 1  # partial overlap
    assert L.w4a16_gemm(A16, A16, A16, None, 1, 8, 64, 32, None, 0, None) == 1
    assert L.w4a16_gemm(A16, A16, A16, A16, 1, 8, 40, 32, None, 0, None) == 1
    assert L.w4a16_gemm(A16, A16, A16, A16, 1, 8, 64, 64, None, 0, None) == 2
    assert L.w4a16_gemm(A16, A16, A16, A16, 1, 8, 64, 32, A16 + 16, 4096, None) == 1  # ws not 256-aligned
    assert L.w4a16_gemm(A16, A16, A16, A16, 0, 8, 64, 32, None, 0, None) == 0   # empty: no launch
    # moe_align: block not a power of two, E too large, capacity too small
    assert L.w4_moe_align(A16, 4, 2, 8, 24, A16, 1024, A16, A16, None) == 1
    assert L.w4_moe_align(A16, 4, 2, 2048, 16, A16, 1 << 20, A16, A16, None) == 1
    assert L.w4_moe_align(A16, 4, 2, 8, 16, A16, 16, A16, A16, None) == 1
    # grouped GEMM: unsupported block size / K, misaligned pointers
    args = [A16, 8, A16, A16, A16, A16, A16, 1024, 16, 128, A16, 3072, 4096, 128, None]
    a = list(args); a[8] = 8
    assert L.w4_moe_w4a16_gemm(*a) == 2
    a = list(args); a[12] = 4096 + 32
    assert L.w4_moe_w4a16_gemm(*a) == 2
    a = list(args); a[10] = MIS
    assert L.w4_moe_w4a16_gemm(*a) == 1
    a = list(args); a[1] = 0
    assert L.w4_moe_w4a16_gemm(*a) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    W = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        w4.w4_fake_quant(W, torch.empty_like(W))


def test_moe_block_size_rule_host_only():
    L = w4.lib()
    assert L.w4_moe_block_size(16, 8, 128) == 16       # 1 slot per expert
    assert L.w4_moe_block_size(768, 8, 128) == 16      # 48: the edge stays 16
    assert L.w4_moe_block_size(769, 8, 128) == 32
    assert L.w4_moe_block_size(1536, 8, 128) == 32     # 96
    assert L.w4_moe_block_size(1537, 8, 128) == 64
    assert L.w4_moe_block_size(0, 8, 128) == 0
    assert L.w4_moe_block_size(16, 0, 128) == 0


def test_moe_glue_validation_host_only():
    L = w4.lib()
    # gating: E out of range, topk > E (twice), T = 0 (nothing to do)
    assert L.w4_moe_gate_topk(A16, 4, 257, 8, A16, A16, None) == 1
    assert L.w4_moe_gate_topk(A16, 4, 8, 9, A16, A16, None) == 1
    assert L.w4_moe_gate_topk(A16, 4, 64, 65, A16, A16, None) == 1
    assert L.w4_moe_gate_topk(A16, 0, 128, 8, A16, A16, None) == 0
    # silu_mul: F not a multiple of 8, misaligned, empty
    assert L.w4_silu_mul(A16, 4, 12, A16, None) == 1
    assert L.w4_silu_mul(MIS, 4, 16, A16, None) == 1
    assert L.w4_silu_mul(A16, 0, 16, A16, None) == 0
    # combine: N not a multiple of 8, topk < 1, misaligned output, empty
    assert L.w4_moe_combine(A16, A16, 4, 8, 12, A16, None) == 1
    assert L.w4_moe_combine(A16, A16, 4, 0, 16, A16, None) == 1
    assert L.w4_moe_combine(A16, A16, 4, 8, 16, MIS, None) == 1
    assert L.w4_moe_combine(A16, A16, 0, 8, 16, A16, None) == 0


def test_qat_gemm_validation_host_only():
    L = w4.lib()
    assert L.w4_qat_gemm(A16, A16, A16, 4, 8, 64, 64, None, 0, None) == 2      # group != 32
    assert L.w4_qat_gemm(A16, A16, A16, 4, 8, 48, 32, None, 0, None) == 1      # K % 32 != 0
    assert L.w4_qat_gemm(A16, A16, A16, 4, 8, 96, 32, None, 0, None) == 2      # K % 64 != 0
    assert L.w4_qat_gemm(MIS, A16, A16, 4, 8, 64, 32, None, 0, None) == 1      # misaligned X
    assert L.w4_qat_gemm(A16, A16, A16, 0, 8, 64, 32, None, 0, None) == 0      # empty: no launch
    assert L.w4_qat_gemm(A16, A16, A16, 4, 8, 64, 32, A16 + 16, 4096, None) == 1  # ws not 256-aligned
    assert L.w4_qat_gemm_dx(A16, A16, A16, 4, 8, 64, 64, None, 0, None) == 2   # group != 32
    assert L.w4_qat_gemm_dx(A16, A16, A16, 4, 12, 64, 32, None, 0, None) == 2  # N % 8 != 0
    assert L.w4_qat_gemm_dx(A16, A16, A16, 0, 8, 64, 32, None, 0, None) == 0   # empty: no launch


def test_zero_point_validation_host_only():
    L = w4.lib()
    assert L.w4_quantize_pack_zp(A16, A16, A16, A16, 4, 64, 64, None) == 2     # group != 32
    assert L.w4_quantize_pack_zp(A16, A16, A16, A16, 4, 48, 32, None) == 1     # K % 32 != 0
    assert L.w4_quantize_pack_zp(A16, A16, A16, None, 4, 64, 32, None) == 1    # Z missing
    assert L.w4_quantize_pack_zp(MIS, A16, A16, A16, 4, 64, 32, None) == 1     # misaligned W
    assert L.w4_quantize_pack_zp(A16, A16, A16, A16, 0, 64, 32, None) == 0     # empty
    assert L.w4_dequant_zp(A16, A16, None, A16, 4, 64, 32, None) == 1
    assert L.w4_dequant_zp(A16, A16, A16, A16, 0, 64, 32, None) == 0
    assert L.w4a16_gemm_zp(A16, A16, A16, A16, A16, 4, 8, 64, 64, None) == 2   # group != 32
    assert L.w4a16_gemm_zp(A16, A16, A16, A16, A16, 4, 8, 48, 32, None) == 1   # K % 32 != 0
    assert L.w4a16_gemm_zp(A16, A16, A16, None, A16, 4, 8, 64, 32, None) == 1  # Z missing
    assert L.w4a16_gemm_zp(A16, A16, A16, A16, MIS, 4, 8, 64, 32, None) == 1   # misaligned Y
    assert L.w4a16_gemm_zp(A16, A16, A16, A16, A16, 0, 8, 64, 32, None) == 0   # empty


def _t(shape, dtype):
    import torch
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("case", ["S_dtype", "S_short", "Y_dtype", "Y_shape", "Wq_cols"])
def test_gemm_binding_checks_every_operand(case):
    """The binding rejects a wrongly typed or sized operand before any pointer
    reaches the library: the C side sizes its bulk copies from M, N and K
    alone, so a short S would be read past its end on the device."""
    import torch
    M, N, K = 4, 64, 256
    X, Wq = _t((M, K), torch.bfloat16), _t((N, K // 8), torch.int32)
    S, Y = _t((N, K // 32), torch.bfloat16), _t((M, N), torch.bfloat16)
    if case == "S_dtype":
        S = _t((N, K // 32), torch.float32)
    elif case == "S_short":
        S = _t((N, K // 64), torch.bfloat16)
    elif case == "Y_dtype":
        Y = _t((M, N), torch.float32)
    elif case == "Y_shape":
        Y = _t((M, N - 1), torch.bfloat16)
    else:
        Wq = _t((N, K // 16), torch.int32)
    for fn in (w4.w4a16_gemm, w4.w4a16_gemm_noalloc):
        with pytest.raises((TypeError, ValueError)) as ei:
            fn(X, Wq, S, Y)
        assert "CUDA tensors" not in str(ei.value), "checked only at the pointer"


def test_quantizer_bindings_check_output_shapes():
    import torch
    W = _t((8, 64), torch.bfloat16)
    with pytest.raises(ValueError):
        w4.w4_quantize_pack(W, _t((8, 8), torch.int32), _t((8, 1), torch.bfloat16))
    with pytest.raises(ValueError):
        w4.w4_fake_quant(W, _t((8, 64), torch.bfloat16), _t((8, 3), torch.bfloat16))
    with pytest.raises(TypeError):
        w4.w4_dequant(_t((8, 8), torch.int32), _t((8, 2), torch.float16), _t((8, 64), torch.bfloat16))
    with pytest.raises(ValueError):
        w4.w4a16_gemm_zp(_t((2, 64), torch.bfloat16), _t((8, 8), torch.int32),
                         _t((8, 2), torch.bfloat16), _t((8, 1), torch.uint8),
                         _t((2, 8), torch.bfloat16))
