"""int4_w4a16_b200 -- group-wise INT4 weight quantization and W4A16 inference on
B200 (sm_100a).

This module is the thin Python binding of ``libw4a16.so`` (C ABI declared in
``include/w4a16.h``).  Each ``w4_*`` function has the name of the C entry point
it calls and only marshals arguments: tensor data pointers, sizes and the
current CUDA stream.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback -- if the library or a CUDA device
is missing, calls raise.

PyTorch is used for device memory and streams only.  BF16 tensors are passed as
``torch.bfloat16``; packed weights as ``torch.int32``.

Sources (page titles): SGLang RL team "INT4 QAT end-to-end" blog (fake
quantization + STE, Fig. 4 packing, moe_align_block_size, MoE operator
fusion); reportify.cn "量化感知训练" [8]-[11], [32], [35]; "量化基础：从 FP32
到 INT4 的压缩艺术" §2.2, §2.4.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "W4Error", "lib", "workspace", "w4a16_gemm_workspace_bytes", "w4_version",
    "w4_device_status", "w4_wait_selftest", "w4_fake_quant", "w4_ste_backward",
    "w4_quantize_pack", "w4_dequant", "w4a16_gemm", "w4_moe_capacity", "w4_moe_align",
    "w4_moe_w4a16_gemm", "w4_moe_w4a16_gemm_silu", "w4_moe_gate_topk", "w4_moe_block_size",
    "w4_silu_mul", "moe_gemm_silu", "w4_qat_gemm", "qat_gemm", "w4_qat_gemm_dx", "qat_gemm_dx",
    "w4_qat_gemm_workspace_bytes",
    "w4_quantize_pack_zp", "w4_dequant_zp", "w4a16_gemm_zp", "quantize_pack_zp", "dequant_zp",
    "gemm_zp",
    "w4_quantize_pack_mxfp4", "w4_dequant_mxfp4", "w4_nvfp4_tensor_scale",
    "w4_quantize_pack_nvfp4", "w4_dequant_nvfp4", "w4a16_gemm_mxfp4", "w4a16_gemm_nvfp4",
    "quantize_pack_mxfp4", "dequant_mxfp4", "gemm_mxfp4", "quantize_pack_nvfp4",
    "dequant_nvfp4", "gemm_nvfp4",
    "w4_moe_combine", "w4_moe_combine_counter_bytes", "w4_moe_w4a16_gemm_combine",
    "moe_gemm_combine", "fake_quant", "quantize_pack", "dequant", "gemm", "moe_align",
    "moe_gate_topk", "silu_mul", "moe_combine",
    "moe_gemm", "FakeInt4STE", "GROUP",
]

GROUP = 32
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a16.so")

_STATUS = {0: "W4_OK", 1: "W4_ERR_INVALID_ARG", 2: "W4_ERR_UNSUPPORTED", 3: "W4_ERR_CUDA",
           4: "W4_ERR_TIMEOUT"}


class W4Error(RuntimeError):
    def __init__(self, fn: str, code: int, cuda_err: int = 0):
        msg = f"{fn} returned {_STATUS.get(code, code)}"
        if code == 3:
            msg += f" (cudaError {cuda_err})"
        super().__init__(msg)
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load libw4a16.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m int4_w4a16_b200.build` "
                "(there is no fallback path)")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in {
            "w4_fake_quant": [_P, _P, _P, _I64, _I64, _INT, _P],
            "w4_ste_backward": [_P, _P, _I64, _P],
            "w4_quantize_pack": [_P, _P, _P, _I64, _I64, _INT, _P],
            "w4_dequant": [_P, _P, _P, _I64, _I64, _INT, _P],
            "w4a16_gemm": [_P, _P, _P, _P, _I64, _I64, _I64, _INT, _P, ctypes.c_size_t, _P],
            "w4a16_gemm_noalloc": [_P, _P, _P, _P, _I64, _I64, _I64, _INT, _P],
            "w4_moe_align": [_P, _I64, _INT, _INT, _INT, _P, _I64, _P, _P, _P],
            "w4_moe_w4a16_gemm": [_P, _INT, _P, _P, _P, _P, _P, _I64, _INT, _I64, _P, _I64,
                                  _I64, _INT, _P],
            "w4_moe_w4a16_gemm_silu": [_P, _INT, _P, _P, _P, _P, _P, _I64, _INT, _I64, _P,
                                       _I64, _I64, _INT, _P],
            "w4_moe_gate_topk": [_P, _I64, _INT, _INT, _P, _P, _P],
            "w4_qat_gemm": [_P, _P, _P, _I64, _I64, _I64, _INT, _P, ctypes.c_size_t, _P],
            "w4_qat_gemm_dx": [_P, _P, _P, _I64, _I64, _I64, _INT, _P, ctypes.c_size_t, _P],
            "w4_quantize_pack_zp": [_P, _P, _P, _P, _I64, _I64, _INT, _P],
            "w4_dequant_zp": [_P, _P, _P, _P, _I64, _I64, _INT, _P],
            "w4a16_gemm_zp": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _INT, _P],
            "w4_quantize_pack_mxfp4": [_P, _P, _P, _I64, _I64, _P],
            "w4_dequant_mxfp4": [_P, _P, _P, _I64, _I64, _P],
            "w4_nvfp4_tensor_scale": [_P, _I64, _P, _P],
            "w4_quantize_pack_nvfp4": [_P, _P, _P, _P, _I64, _I64, _P],
            "w4_dequant_nvfp4": [_P, _P, ctypes.c_float, _P, _I64, _I64, _P],
            "w4a16_gemm_mxfp4": [_P, _P, _P, _P, _I64, _I64, _I64, _P],
            "w4a16_gemm_nvfp4": [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, _P],
            "w4_silu_mul": [_P, _I64, _I64, _P, _P],
            "w4_moe_combine": [_P, _P, _I64, _INT, _I64, _P, _P],
            "w4_moe_w4a16_gemm_combine": [_P, _P, _P, _P, _P, _P, _I64, _INT, _INT, _P, _P, _P,
                                          _P, _I64, _I64, _I64, _INT, _P],
            "w4_device_status": [_P],
            "w4_wait_selftest": [ctypes.c_uint32, _P],
        }.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.w4a16_gemm_workspace_bytes.argtypes = [_I64, _I64, _I64]
        L.w4a16_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.w4_qat_gemm_workspace_bytes.argtypes = [_I64, _I64, _I64]
        L.w4_qat_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.w4_moe_capacity.argtypes = [_I64, _INT, _INT, _INT]
        L.w4_moe_capacity.restype = ctypes.c_int64
        L.w4_moe_block_size.argtypes = [_I64, _INT, _INT]
        L.w4_moe_combine_counter_bytes.argtypes = [_I64, _I64]
        L.w4_moe_combine_counter_bytes.restype = ctypes.c_size_t
        L.w4_moe_block_size.restype = ctypes.c_int
        L.w4_version.restype = ctypes.c_int
        L.w4_last_cuda_error.restype = ctypes.c_int
        L.w4_status_string.argtypes = [_INT]
        L.w4_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise W4Error(fn, rc, lib().w4_last_cuda_error() if rc == 3 else 0)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libw4a16 takes CUDA tensors (device memory)")
    if not t.is_contiguous():
        raise ValueError("libw4a16 takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _dtype(t: torch.Tensor, dt: torch.dtype, what: str) -> None:
    if t.dtype != dt:
        raise TypeError(f"{what} must be {dt}, got {t.dtype}")


def _arg(t: torch.Tensor, dt: torch.dtype, shape: tuple, what: str) -> None:
    """dtype and exact shape: the C side sizes its bulk copies from the
    integer arguments alone, so a smaller buffer would be read or written
    past its end on the device."""
    _dtype(t, dt, what)
    if tuple(t.shape) != tuple(int(d) for d in shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _group_cols(K: int, group: int, what: str) -> int:
    if group <= 0 or K % group:
        raise ValueError(f"{what}: K = {K} is not a multiple of the group size {group}")
    return K // group


# ---------------------------------------------------------------------------
# C-ABI calls (same names as include/w4a16.h)
# ---------------------------------------------------------------------------

def w4_version() -> int:
    return int(lib().w4_version())


def w4_device_status(stream=None) -> None:
    """Synchronize the stream and raise if a kernel gave up a bounded wait."""
    _check("w4_device_status", lib().w4_device_status(_stream(stream)))


def w4_wait_selftest(limit_us: int, stream=None) -> None:
    """Launch the bounded-wait self-test (see include/w4a16.h); the next
    w4_device_status() raises W4Error with status W4_ERR_TIMEOUT."""
    _check("w4_wait_selftest", lib().w4_wait_selftest(int(limit_us), _stream(stream)))


def w4_fake_quant(W, Wdq, S=None, group: int = GROUP, stream=None) -> None:
    _dtype(W, torch.bfloat16, "W")
    rows, K = W.shape
    _arg(Wdq, torch.bfloat16, (rows, K), "Wdq")
    if S is not None:
        _arg(S, torch.bfloat16, (rows, _group_cols(K, group, "w4_fake_quant")), "S")
    _check("w4_fake_quant", lib().w4_fake_quant(_ptr(W), _ptr(Wdq), _ptr(S), rows, K, group,
                                                _stream(stream)))


def w4_ste_backward(dWdq, dW, stream=None) -> None:
    _dtype(dWdq, torch.bfloat16, "dWdq")
    _dtype(dW, torch.bfloat16, "dW")
    if dW.numel() != dWdq.numel():
        raise ValueError("dW and dWdq must have the same number of elements")
    _check("w4_ste_backward", lib().w4_ste_backward(_ptr(dWdq), _ptr(dW), dWdq.numel(),
                                                    _stream(stream)))


def w4_quantize_pack(W, Wq, S, group: int = GROUP, stream=None) -> None:
    _dtype(W, torch.bfloat16, "W")
    rows, K = W.shape
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.bfloat16, (rows, _group_cols(K, group, "w4_quantize_pack")), "S")
    _check("w4_quantize_pack", lib().w4_quantize_pack(_ptr(W), _ptr(Wq), _ptr(S), rows, K,
                                                      group, _stream(stream)))


def w4_dequant(Wq, S, Wdq, group: int = GROUP, stream=None) -> None:
    _dtype(Wdq, torch.bfloat16, "Wdq")
    rows, K = Wdq.shape
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.bfloat16, (rows, _group_cols(K, group, "w4_dequant")), "S")
    _check("w4_dequant", lib().w4_dequant(_ptr(Wq), _ptr(S), _ptr(Wdq), rows, K, group,
                                          _stream(stream)))


_WORKSPACE = {}


def workspace(device, nbytes: int) -> torch.Tensor:
    """A zeroed per-device scratch buffer of at least nbytes for the split GEMM
    schedule (the kernels leave it zeroed after every call)."""
    idx = torch.device(device).index
    t = _WORKSPACE.get(idx)
    if t is None or t.numel() < nbytes:
        t = torch.zeros(max(int(nbytes), 1 << 20), dtype=torch.uint8, device=device)
        _WORKSPACE[idx] = t
    return t


def _gemm_args(X, Wq, S, Y, group: int, fn: str):
    """X [M, K] bf16, Wq [N, K/8] int32, S [N, K/group] bf16, Y [M, N] bf16."""
    _dtype(X, torch.bfloat16, "X")
    _dtype(Wq, torch.int32, "Wq")
    M, K = X.shape
    N = Wq.shape[0]
    _arg(Wq, torch.int32, (N, K // 8), "Wq")
    _arg(S, torch.bfloat16, (N, _group_cols(K, group, fn)), "S")
    _arg(Y, torch.bfloat16, (M, N), "Y")
    return M, K, N


def w4a16_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().w4a16_gemm_workspace_bytes(M, N, K))


def w4a16_gemm(X, Wq, S, Y, group: int = GROUP, ws="auto", stream=None) -> None:
    """ws: "auto" (the module's zeroed per-device buffer), None (unsplit
    schedule), or a zeroed uint8 CUDA tensor."""
    M, K, N = _gemm_args(X, Wq, S, Y, group, "w4a16_gemm")
    if isinstance(ws, str):
        need = w4a16_gemm_workspace_bytes(M, N, K)
        ws = workspace(X.device, need) if need > 0 else None
    wptr, wbytes = (_ptr(ws), ws.numel() * ws.element_size()) if ws is not None else (None, 0)
    _check("w4a16_gemm", lib().w4a16_gemm(_ptr(X), _ptr(Wq), _ptr(S), _ptr(Y), M, N, K, group,
                                          wptr, wbytes, _stream(stream)))


def w4a16_gemm_noalloc(X, Wq, S, Y, group: int = GROUP, stream=None) -> None:
    """w4a16_gemm without any workspace argument or allocation: the library uses
    a fixed 8 MiB scratch array of its own per device (see include/w4a16.h for
    who needs this and its limits)."""
    M, K, N = _gemm_args(X, Wq, S, Y, group, "w4a16_gemm_noalloc")
    _check("w4a16_gemm_noalloc", lib().w4a16_gemm_noalloc(_ptr(X), _ptr(Wq), _ptr(S), _ptr(Y),
                                                          M, N, K, group, _stream(stream)))


def w4_moe_capacity(T: int, topk: int, E: int, block: int) -> int:
    return int(lib().w4_moe_capacity(T, topk, E, block))


def w4_moe_align(topk_ids, E: int, block: int, sorted_ids, expert_ids, num_post_pad,
                 stream=None) -> None:
    _dtype(topk_ids, torch.int32, "topk_ids")
    T, topk = topk_ids.shape
    _dtype(sorted_ids, torch.int32, "sorted_ids")
    cap = sorted_ids.numel()
    _arg(expert_ids, torch.int32, (cap // block if block > 0 else 0,), "expert_ids")
    _arg(num_post_pad, torch.int32, (1,), "num_post_pad")
    _check("w4_moe_align", lib().w4_moe_align(_ptr(topk_ids), T, topk, E, block,
                                              _ptr(sorted_ids), sorted_ids.numel(),
                                              _ptr(expert_ids), _ptr(num_post_pad),
                                              _stream(stream)))


def _moe_args(A, a_row_div, S, sorted_ids, expert_ids, num_post_pad, block, num_slots, E, N,
              K, fn):
    _dtype(A, torch.bfloat16, "A")
    if A.dim() != 2 or A.shape[1] != K:
        raise ValueError(f"A must be [rows, {K}], got {tuple(A.shape)}")
    if a_row_div <= 0 or A.shape[0] * a_row_div < num_slots:
        raise ValueError(f"A has {A.shape[0]} rows; slot / {a_row_div} must index them for "
                         f"{num_slots} slots")
    _arg(S, torch.bfloat16, (E, N, _group_cols(K, GROUP, fn)), "S")
    _dtype(sorted_ids, torch.int32, "sorted_ids")
    _arg(expert_ids, torch.int32, (sorted_ids.numel() // block if block > 0 else 0,),
         "expert_ids")
    _arg(num_post_pad, torch.int32, (1,), "num_post_pad")


def w4_moe_w4a16_gemm(A, a_row_div: int, Wq, S, sorted_ids, expert_ids, num_post_pad,
                      block: int, num_slots: int, C, stream=None) -> None:
    _dtype(Wq, torch.int32, "Wq")
    E, N, K8 = Wq.shape
    _moe_args(A, a_row_div, S, sorted_ids, expert_ids, num_post_pad, block, num_slots, E, N,
              K8 * 8, "w4_moe_w4a16_gemm")
    _arg(C, torch.bfloat16, (num_slots, N), "C")
    _check("w4_moe_w4a16_gemm", lib().w4_moe_w4a16_gemm(
        _ptr(A), a_row_div, _ptr(Wq), _ptr(S), _ptr(sorted_ids), _ptr(expert_ids),
        _ptr(num_post_pad), sorted_ids.numel(), block, num_slots, _ptr(C), N, K8 * 8, E,
        _stream(stream)))


def w4_moe_combine_counter_bytes(T: int, N: int) -> int:
    return int(lib().w4_moe_combine_counter_bytes(T, N))


def w4_moe_w4a16_gemm_combine(A, Wq, S, sorted_ids, expert_ids, num_post_pad, block: int, w,
                              C, counters, out, stream=None) -> None:
    """Down projection with the weighted top-k combine fused: A [T*topk, K], w
    [T, topk] fp32, C [T*topk, N], counters uint8 (zeroed, w4_moe_combine_counter_bytes),
    out [T, N]."""
    _dtype(Wq, torch.int32, "Wq")
    E, N, K8 = Wq.shape
    _dtype(w, torch.float32, "w")
    T, topk = w.shape
    num_slots = T * topk
    _moe_args(A, 1, S, sorted_ids, expert_ids, num_post_pad, block, num_slots, E, N, K8 * 8,
              "w4_moe_w4a16_gemm_combine")
    _arg(C, torch.bfloat16, (num_slots, N), "C")
    _arg(out, torch.bfloat16, (T, N), "out")
    _dtype(counters, torch.uint8, "counters")
    if counters.numel() < w4_moe_combine_counter_bytes(T, N):
        raise ValueError("counters is smaller than w4_moe_combine_counter_bytes(T, N)")
    _check("w4_moe_w4a16_gemm_combine", lib().w4_moe_w4a16_gemm_combine(
        _ptr(A), _ptr(Wq), _ptr(S), _ptr(sorted_ids), _ptr(expert_ids), _ptr(num_post_pad),
        sorted_ids.numel(), block, topk, _ptr(w), _ptr(C), _ptr(counters), _ptr(out), T, N,
        K8 * 8, E, _stream(stream)))


def w4_moe_w4a16_gemm_silu(A, a_row_div: int, Wq, S, sorted_ids, expert_ids, num_post_pad,
                           block: int, num_slots: int, H, stream=None) -> None:
    """gate_up grouped GEMM with SiLU*up fused: Wq [E, 2F, K/8]; H [num_slots, F]."""
    _dtype(Wq, torch.int32, "Wq")
    E, N2, K8 = Wq.shape
    _moe_args(A, a_row_div, S, sorted_ids, expert_ids, num_post_pad, block, num_slots, E, N2,
              K8 * 8, "w4_moe_w4a16_gemm_silu")
    _arg(H, torch.bfloat16, (num_slots, N2 // 2), "H")
    _check("w4_moe_w4a16_gemm_silu", lib().w4_moe_w4a16_gemm_silu(
        _ptr(A), a_row_div, _ptr(Wq), _ptr(S), _ptr(sorted_ids), _ptr(expert_ids),
        _ptr(num_post_pad), sorted_ids.numel(), block, num_slots, _ptr(H), N2 // 2, K8 * 8, E,
        _stream(stream)))


def _ws_args(ws, need: int, device):
    """ws: "auto" (the module's zeroed per-device buffer), None, or a zeroed
    uint8 CUDA tensor -> (pointer, bytes)."""
    if isinstance(ws, str):
        ws = workspace(device, need) if need > 0 else None
    return (_ptr(ws), ws.numel() * ws.element_size()) if ws is not None else (None, 0)


def w4_qat_gemm_workspace_bytes(M: int, rows: int, contraction: int) -> int:
    return int(lib().w4_qat_gemm_workspace_bytes(M, rows, contraction))


def w4_qat_gemm(X, W, Y, group: int = GROUP, ws="auto", stream=None) -> None:
    """Y = X . fake_quant(W)^T, the QDQ fused into the GEMM's weight prologue."""
    _dtype(X, torch.bfloat16, "X")
    M, K = X.shape
    _dtype(W, torch.bfloat16, "W")
    N = W.shape[0]
    _arg(W, torch.bfloat16, (N, K), "W")
    _arg(Y, torch.bfloat16, (M, N), "Y")
    wptr, wbytes = _ws_args(ws, w4_qat_gemm_workspace_bytes(M, N, K), X.device)
    _check("w4_qat_gemm", lib().w4_qat_gemm(_ptr(X), _ptr(W), _ptr(Y), M, N, K, group, wptr,
                                            wbytes, _stream(stream)))


def w4_qat_gemm_dx(dY, W, dX, group: int = GROUP, ws="auto", stream=None) -> None:
    """dX = dY . fake_quant(W), the QDQ fused into the GEMM's weight prologue."""
    _dtype(dY, torch.bfloat16, "dY")
    M, N = dY.shape
    _dtype(W, torch.bfloat16, "W")
    K = W.shape[1]
    _arg(W, torch.bfloat16, (N, K), "W")
    _arg(dX, torch.bfloat16, (M, K), "dX")
    wptr, wbytes = _ws_args(ws, w4_qat_gemm_workspace_bytes(M, K, N), dY.device)
    _check("w4_qat_gemm_dx", lib().w4_qat_gemm_dx(_ptr(dY), _ptr(W), _ptr(dX), M, N, K, group,
                                                  wptr, wbytes, _stream(stream)))


def w4_quantize_pack_zp(W, Wq, S, Z, group: int = GROUP, stream=None) -> None:
    """Asymmetric groups: unsigned codes Wq, BF16 scales S, uint8 zero points Z."""
    _dtype(W, torch.bfloat16, "W")
    rows, K = W.shape
    G = _group_cols(K, group, "w4_quantize_pack_zp")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.bfloat16, (rows, G), "S")
    _arg(Z, torch.uint8, (rows, G), "Z")
    _check("w4_quantize_pack_zp", lib().w4_quantize_pack_zp(_ptr(W), _ptr(Wq), _ptr(S), _ptr(Z),
                                                            rows, K, group, _stream(stream)))


def w4_dequant_zp(Wq, S, Z, Wdq, group: int = GROUP, stream=None) -> None:
    _dtype(Wdq, torch.bfloat16, "Wdq")
    rows, K = Wdq.shape
    G = _group_cols(K, group, "w4_dequant_zp")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.bfloat16, (rows, G), "S")
    _arg(Z, torch.uint8, (rows, G), "Z")
    _check("w4_dequant_zp", lib().w4_dequant_zp(_ptr(Wq), _ptr(S), _ptr(Z), _ptr(Wdq), rows, K,
                                                group, _stream(stream)))


def w4a16_gemm_zp(X, Wq, S, Z, Y, group: int = GROUP, stream=None) -> None:
    M, K, N = _gemm_args(X, Wq, S, Y, group, "w4a16_gemm_zp")
    _arg(Z, torch.uint8, (N, K // group), "Z")
    _check("w4a16_gemm_zp", lib().w4a16_gemm_zp(_ptr(X), _ptr(Wq), _ptr(S), _ptr(Z), _ptr(Y),
                                                M, N, K, group, _stream(stream)))


def _fp4_cols(K: int, what: str) -> None:
    if K <= 0 or K % 32:
        raise ValueError(f"{what}: K = {K} is not a positive multiple of 32")


def w4_quantize_pack_mxfp4(W, Wq, E, stream=None) -> None:
    """MXFP4: E2M1 codes Wq [rows, K/8] int32 and E8M0 exponents E [rows, K/32] uint8."""
    _dtype(W, torch.bfloat16, "W")
    rows, K = W.shape
    _fp4_cols(K, "w4_quantize_pack_mxfp4")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(E, torch.uint8, (rows, K // 32), "E")
    _check("w4_quantize_pack_mxfp4", lib().w4_quantize_pack_mxfp4(_ptr(W), _ptr(Wq), _ptr(E),
                                                                  rows, K, _stream(stream)))


def w4_dequant_mxfp4(Wq, E, Wdq, stream=None) -> None:
    _dtype(Wdq, torch.bfloat16, "Wdq")
    rows, K = Wdq.shape
    _fp4_cols(K, "w4_dequant_mxfp4")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(E, torch.uint8, (rows, K // 32), "E")
    _check("w4_dequant_mxfp4", lib().w4_dequant_mxfp4(_ptr(Wq), _ptr(E), _ptr(Wdq), rows, K,
                                                      _stream(stream)))


def w4_nvfp4_tensor_scale(W, g, stream=None) -> None:
    """g: a one-element float32 CUDA tensor, set to fl32(max|W| / 2688) (1 if W == 0)."""
    _dtype(W, torch.bfloat16, "W")
    _arg(g, torch.float32, (1,), "g")
    _check("w4_nvfp4_tensor_scale", lib().w4_nvfp4_tensor_scale(_ptr(W), W.numel(), _ptr(g),
                                                                _stream(stream)))


def w4_quantize_pack_nvfp4(W, g, Wq, S, stream=None) -> None:
    """NVFP4 under the device tensor scale g: codes Wq [rows, K/8], E4M3 scales S [rows, K/16]."""
    _dtype(W, torch.bfloat16, "W")
    rows, K = W.shape
    _fp4_cols(K, "w4_quantize_pack_nvfp4")
    _arg(g, torch.float32, (1,), "g")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.uint8, (rows, K // 16), "S")
    _check("w4_quantize_pack_nvfp4", lib().w4_quantize_pack_nvfp4(_ptr(W), _ptr(g), _ptr(Wq),
                                                                  _ptr(S), rows, K,
                                                                  _stream(stream)))


def w4_dequant_nvfp4(Wq, S, g: float, Wdq, stream=None) -> None:
    _dtype(Wdq, torch.bfloat16, "Wdq")
    rows, K = Wdq.shape
    _fp4_cols(K, "w4_dequant_nvfp4")
    _arg(Wq, torch.int32, (rows, K // 8), "Wq")
    _arg(S, torch.uint8, (rows, K // 16), "S")
    _check("w4_dequant_nvfp4", lib().w4_dequant_nvfp4(_ptr(Wq), _ptr(S), float(g), _ptr(Wdq),
                                                      rows, K, _stream(stream)))


def _fp4_gemm_args(X, Wq, Y, what: str):
    _dtype(X, torch.bfloat16, "X")
    M, K = X.shape
    _fp4_cols(K, what)
    _dtype(Wq, torch.int32, "Wq")
    N = Wq.shape[0]
    _arg(Wq, torch.int32, (N, K // 8), "Wq")
    _arg(Y, torch.bfloat16, (M, N), "Y")
    return M, K, N


def w4a16_gemm_mxfp4(X, Wq, E, Y, stream=None) -> None:
    M, K, N = _fp4_gemm_args(X, Wq, Y, "w4a16_gemm_mxfp4")
    _arg(E, torch.uint8, (N, K // 32), "E")
    _check("w4a16_gemm_mxfp4", lib().w4a16_gemm_mxfp4(_ptr(X), _ptr(Wq), _ptr(E), _ptr(Y), M, N,
                                                      K, _stream(stream)))


def w4a16_gemm_nvfp4(X, Wq, S, g: float, Y, stream=None) -> None:
    M, K, N = _fp4_gemm_args(X, Wq, Y, "w4a16_gemm_nvfp4")
    _arg(S, torch.uint8, (N, K // 16), "S")
    _check("w4a16_gemm_nvfp4", lib().w4a16_gemm_nvfp4(_ptr(X), _ptr(Wq), _ptr(S), float(g),
                                                      _ptr(Y), M, N, K, _stream(stream)))


def w4_moe_gate_topk(logits, topk: int, topk_ids, topk_weights, stream=None) -> None:
    _dtype(logits, torch.float32, "logits")
    T, E = logits.shape
    _arg(topk_ids, torch.int32, (T, topk), "topk_ids")
    _arg(topk_weights, torch.float32, (T, topk), "topk_weights")
    _check("w4_moe_gate_topk", lib().w4_moe_gate_topk(_ptr(logits), T, E, topk, _ptr(topk_ids),
                                                      _ptr(topk_weights), _stream(stream)))


def w4_moe_block_size(T: int, topk: int, E: int) -> int:
    return int(lib().w4_moe_block_size(T, topk, E))


def w4_silu_mul(gate_up, h, stream=None) -> None:
    _dtype(gate_up, torch.bfloat16, "gate_up")
    S, F2 = gate_up.shape
    _arg(h, torch.bfloat16, (S, F2 // 2), "h")
    _check("w4_silu_mul", lib().w4_silu_mul(_ptr(gate_up), S, F2 // 2, _ptr(h), _stream(stream)))


def w4_moe_combine(D, w, out, stream=None) -> None:
    _dtype(w, torch.float32, "w")
    T, topk = w.shape
    _dtype(D, torch.bfloat16, "D")
    _arg(D, torch.bfloat16, (T * topk, D.shape[1]), "D")
    _arg(out, torch.bfloat16, (T, D.shape[1]), "out")
    _check("w4_moe_combine", lib().w4_moe_combine(_ptr(D), _ptr(w), T, topk, D.shape[1],
                                                  _ptr(out), _stream(stream)))


# ---------------------------------------------------------------------------
# Allocating conveniences (outputs from torch.empty on the input's device)
# ---------------------------------------------------------------------------

def fake_quant(W: torch.Tensor, want_scales: bool = False):
    rows, K = W.shape
    Wdq = torch.empty_like(W)
    S = torch.empty((rows, K // GROUP), dtype=torch.bfloat16, device=W.device) if want_scales else None
    w4_fake_quant(W, Wdq, S)
    return (Wdq, S) if want_scales else Wdq


def quantize_pack(W: torch.Tensor):
    rows, K = W.shape
    Wq = torch.empty((rows, K // 8), dtype=torch.int32, device=W.device)
    S = torch.empty((rows, K // GROUP), dtype=torch.bfloat16, device=W.device)
    w4_quantize_pack(W, Wq, S)
    return Wq, S


def dequant(Wq: torch.Tensor, S: torch.Tensor) -> torch.Tensor:
    rows, K8 = Wq.shape
    Wdq = torch.empty((rows, K8 * 8), dtype=torch.bfloat16, device=Wq.device)
    w4_dequant(Wq, S, Wdq)
    return Wdq


def quantize_pack_zp(W: torch.Tensor):
    rows, K = W.shape
    Wq = torch.empty((rows, K // 8), dtype=torch.int32, device=W.device)
    S = torch.empty((rows, K // GROUP), dtype=torch.bfloat16, device=W.device)
    Z = torch.empty((rows, K // GROUP), dtype=torch.uint8, device=W.device)
    w4_quantize_pack_zp(W, Wq, S, Z)
    return Wq, S, Z


def dequant_zp(Wq: torch.Tensor, S: torch.Tensor, Z: torch.Tensor) -> torch.Tensor:
    rows, K8 = Wq.shape
    Wdq = torch.empty((rows, K8 * 8), dtype=torch.bfloat16, device=Wq.device)
    w4_dequant_zp(Wq, S, Z, Wdq)
    return Wdq


def gemm_zp(X: torch.Tensor, Wq: torch.Tensor, S: torch.Tensor, Z: torch.Tensor) -> torch.Tensor:
    Y = torch.empty((X.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device=X.device)
    w4a16_gemm_zp(X, Wq, S, Z, Y)
    return Y


def quantize_pack_mxfp4(W: torch.Tensor):
    rows, K = W.shape
    Wq = torch.empty((rows, K // 8), dtype=torch.int32, device=W.device)
    E = torch.empty((rows, K // 32), dtype=torch.uint8, device=W.device)
    w4_quantize_pack_mxfp4(W, Wq, E)
    return Wq, E


def dequant_mxfp4(Wq: torch.Tensor, E: torch.Tensor) -> torch.Tensor:
    rows, K8 = Wq.shape
    Wdq = torch.empty((rows, K8 * 8), dtype=torch.bfloat16, device=Wq.device)
    w4_dequant_mxfp4(Wq, E, Wdq)
    return Wdq


def gemm_mxfp4(X: torch.Tensor, Wq: torch.Tensor, E: torch.Tensor) -> torch.Tensor:
    Y = torch.empty((X.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device=X.device)
    w4a16_gemm_mxfp4(X, Wq, E, Y)
    return Y


def quantize_pack_nvfp4(W: torch.Tensor):
    """Returns (Wq, S, g) with g a one-element float32 device tensor."""
    rows, K = W.shape
    g = torch.empty((1,), dtype=torch.float32, device=W.device)
    Wq = torch.empty((rows, K // 8), dtype=torch.int32, device=W.device)
    S = torch.empty((rows, K // 16), dtype=torch.uint8, device=W.device)
    w4_nvfp4_tensor_scale(W, g)
    w4_quantize_pack_nvfp4(W, g, Wq, S)
    return Wq, S, g


def dequant_nvfp4(Wq: torch.Tensor, S: torch.Tensor, g: float) -> torch.Tensor:
    rows, K8 = Wq.shape
    Wdq = torch.empty((rows, K8 * 8), dtype=torch.bfloat16, device=Wq.device)
    w4_dequant_nvfp4(Wq, S, g, Wdq)
    return Wdq


def gemm_nvfp4(X: torch.Tensor, Wq: torch.Tensor, S: torch.Tensor, g: float) -> torch.Tensor:
    Y = torch.empty((X.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device=X.device)
    w4a16_gemm_nvfp4(X, Wq, S, g, Y)
    return Y


def gemm(X: torch.Tensor, Wq: torch.Tensor, S: torch.Tensor, ws="auto") -> torch.Tensor:
    Y = torch.empty((X.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device=X.device)
    w4a16_gemm(X, Wq, S, Y, ws=ws)
    return Y


def moe_align(topk_ids: torch.Tensor, E: int, block: int):
    T, topk = topk_ids.shape
    cap = w4_moe_capacity(T, topk, E, block)
    dev = topk_ids.device
    sorted_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    expert_ids = torch.empty(cap // block, dtype=torch.int32, device=dev)
    npp = torch.empty(4, dtype=torch.int32, device=dev)[:1]
    w4_moe_align(topk_ids, E, block, sorted_ids, expert_ids, npp)
    return sorted_ids, expert_ids, npp


def moe_gemm(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, block, num_slots,
             C=None):
    if C is None:
        C = torch.empty((num_slots, Wq.shape[1]), dtype=torch.bfloat16, device=A.device)
    w4_moe_w4a16_gemm(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, block,
                      num_slots, C)
    return C


def moe_gemm_combine(H, Wq, S, sorted_ids, expert_ids, num_post_pad, block, w, counters,
                     C=None, out=None):
    """Returns (C, out): the down projection's slot rows and their weighted combine."""
    T, topk = w.shape
    if C is None:
        C = torch.empty((T * topk, Wq.shape[1]), dtype=torch.bfloat16, device=H.device)
    if out is None:
        out = torch.empty((T, Wq.shape[1]), dtype=torch.bfloat16, device=H.device)
    w4_moe_w4a16_gemm_combine(H, Wq, S, sorted_ids, expert_ids, num_post_pad, block, w, C,
                              counters, out)
    return C, out


def moe_gemm_silu(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, block, num_slots,
                  H=None):
    if H is None:
        H = torch.empty((num_slots, Wq.shape[1] // 2), dtype=torch.bfloat16, device=A.device)
    w4_moe_w4a16_gemm_silu(A, a_row_div, Wq, S, sorted_ids, expert_ids, num_post_pad, block,
                           num_slots, H)
    return H


def qat_gemm(X: torch.Tensor, W: torch.Tensor, ws="auto") -> torch.Tensor:
    Y = torch.empty((X.shape[0], W.shape[0]), dtype=torch.bfloat16, device=X.device)
    w4_qat_gemm(X, W, Y, ws=ws)
    return Y


def qat_gemm_dx(dY: torch.Tensor, W: torch.Tensor, ws="auto") -> torch.Tensor:
    dX = torch.empty((dY.shape[0], W.shape[1]), dtype=torch.bfloat16, device=dY.device)
    w4_qat_gemm_dx(dY, W, dX, ws=ws)
    return dX


def moe_gate_topk(logits: torch.Tensor, topk: int):
    T = logits.shape[0]
    ids = torch.empty((T, topk), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, topk), dtype=torch.float32, device=logits.device)
    w4_moe_gate_topk(logits, topk, ids, w)
    return ids, w


def silu_mul(gate_up: torch.Tensor) -> torch.Tensor:
    h = torch.empty((gate_up.shape[0], gate_up.shape[1] // 2), dtype=torch.bfloat16,
                    device=gate_up.device)
    w4_silu_mul(gate_up, h)
    return h


def moe_combine(D: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    out = torch.empty((w.shape[0], D.shape[1]), dtype=torch.bfloat16, device=D.device)
    w4_moe_combine(D, w, out)
    return out


class FakeInt4STE(torch.autograd.Function):
    """Fake INT4 quantization with a straight-through estimator.

    Forward: Wdq = w4_fake_quant(W) (group-32 QDQ, BF16 in and out).
    Backward: the gradient passes through the rounding unchanged (identity,
    zero-copy), as in the INT4 QAT blog's _FakeInt4QuantizationSTE.
    """

    @staticmethod
    def forward(ctx, W):
        return fake_quant(W.contiguous())

    @staticmethod
    def backward(ctx, grad_out):
        return grad_out
