"""CPU oracle for group-wise INT4 quantization and W4A16 inference.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``int4_w4a16_b200``) never imports it and shares no
code with it; the CUDA library fails loudly instead of falling back here.

This module is a ctypes binding over ``w4_oracle.c`` (the plain definitions,
with citations) plus numpy conveniences.  Arrays are numpy; BF16 values travel
as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


GCC_FLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
             "-fno-fast-math", "-ffp-contract=off"]


def compile_source(src: str, out: str) -> str:
    subprocess.run(["gcc", *GCC_FLAGS, "-o", out, src, "-lm"], check=True)
    return out


def build(force: bool = False) -> str:
    """Compile ``w4_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


def load_library(path: str) -> ctypes.CDLL:
    """Load an oracle shared library built from ``w4_oracle.c`` and declare its
    signatures (tests also load deliberately mutated copies through this)."""
    L = ctypes.CDLL(path)
    L.w4o_f32_from_bf16.restype = ctypes.c_float
    L.w4o_f32_from_bf16.argtypes = [ctypes.c_uint16]
    L.w4o_bf16_from_f32.restype = ctypes.c_uint16
    L.w4o_bf16_from_f32.argtypes = [ctypes.c_float]
    L.w4o_set_threads.argtypes = [ctypes.c_int]
    L.w4o_get_threads.restype = ctypes.c_int
    L.w4o_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.w4o_fake_quant.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.w4o_ste_backward.argtypes = [_P, _I64, _P]
    L.w4o_pack8_u.restype = ctypes.c_int32
    L.w4o_pack8_u.argtypes = [_P]
    L.w4o_unpack8_u.argtypes = [ctypes.c_int32, _P]
    L.w4o_pack8.restype = ctypes.c_int32
    L.w4o_pack8.argtypes = [_P]
    L.w4o_unpack8.argtypes = [ctypes.c_int32, _P]
    L.w4o_pack.argtypes = [_P, _I64, _P]
    L.w4o_unpack.argtypes = [_P, _I64, _P]
    L.w4o_quantize_pack.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.w4o_dequant.argtypes = [_P, _P, _I64, _I64, _I64, _P]
    L.w4o_symmetric_quantize_f64.argtypes = [_P, _I64, _I64, ctypes.c_int, _P, _P]
    L.w4o_gemm.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P]
    L.w4o_w4a16_gemm.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P]
    L.w4o_quantize_zp.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
    L.w4o_quantize_pack_zp.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
    L.w4o_dequant_zp.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P]
    L.w4o_e2m1_value.restype = ctypes.c_double
    L.w4o_e2m1_value.argtypes = [ctypes.c_uint8]
    L.w4o_e2m1_encode.restype = ctypes.c_uint8
    L.w4o_e2m1_encode.argtypes = [ctypes.c_double]
    L.w4o_e4m3_value.restype = ctypes.c_double
    L.w4o_e4m3_value.argtypes = [ctypes.c_uint8]
    L.w4o_e4m3_encode.restype = ctypes.c_uint8
    L.w4o_e4m3_encode.argtypes = [ctypes.c_double]
    L.w4o_quantize_mxfp4.argtypes = [_P, _I64, _I64, _P, _P]
    L.w4o_dequant_mxfp4.argtypes = [_P, _P, _I64, _I64, _P]
    L.w4o_quantize_nvfp4.argtypes = [_P, _I64, _I64, _P, _P, _P]
    L.w4o_dequant_nvfp4.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P]
    L.w4o_moe_align.restype = ctypes.c_int
    L.w4o_moe_align.argtypes = [_P, _I64, _I64, _I64, _I64, _P, _I64, _P, _P]
    L.w4o_moe_gemm.argtypes = [_P, _I64, _P, _P, _P, _I64, _I64, _I64, _I64,
                               _I64, _P, _P]
    L.w4o_moe_gate_topk.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.w4o_moe_combine.argtypes = [_P, _P, _I64, _I64, _I64, _P]
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = load_library(_LIB_PATH)
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, f"expected raw BF16 bits (uint16), got {a.dtype}"
    return a


def set_threads(n: int) -> None:
    lib().w4o_set_threads(int(n))


def get_threads() -> int:
    return int(lib().w4o_get_threads())


# ---- scalar conversions ---------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def bf16_from_f32_scalar(x: float) -> int:
    return int(lib().w4o_bf16_from_f32(ctypes.c_float(x)))


# ---- quantization ---------------------------------------------------------

def quantize(W: np.ndarray, group: int = 32):
    """(q int8 [rows, K], S bf16-bits [rows, K/group])."""
    W = _u16(W)
    rows, K = W.shape
    q = np.empty((rows, K), np.int8)
    S = np.empty((rows, K // group), np.uint16)
    lib().w4o_quantize(_ptr(W), rows, K, group, _ptr(q), _ptr(S))
    return q, S


def fake_quant(W: np.ndarray, group: int = 32):
    """(Wdq bf16-bits [rows, K], S bf16-bits [rows, K/group])."""
    W = _u16(W)
    rows, K = W.shape
    Wdq = np.empty((rows, K), np.uint16)
    S = np.empty((rows, K // group), np.uint16)
    lib().w4o_fake_quant(_ptr(W), rows, K, group, _ptr(Wdq), _ptr(S))
    return Wdq, S


def ste_backward(dWdq: np.ndarray) -> np.ndarray:
    dWdq = _u16(dWdq)
    dW = np.empty_like(dWdq)
    lib().w4o_ste_backward(_ptr(dWdq), dWdq.size, _ptr(dW))
    return dW


def pack(q: np.ndarray) -> np.ndarray:
    """int8 codes (last dim a multiple of 8) -> int32 words."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    words = np.empty(q.shape[:-1] + (q.shape[-1] // 8,), np.int32)
    lib().w4o_pack(_ptr(q), q.size, _ptr(words))
    return words


def unpack(words: np.ndarray) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.int32)
    q = np.empty(words.shape[:-1] + (words.shape[-1] * 8,), np.int8)
    lib().w4o_unpack(_ptr(words), q.size, _ptr(q))
    return q


def quantize_pack(W: np.ndarray, group: int = 32):
    """(Wq int32 [rows, K/8], S bf16-bits [rows, K/group])."""
    W = _u16(W)
    rows, K = W.shape
    Wq = np.empty((rows, K // 8), np.int32)
    S = np.empty((rows, K // group), np.uint16)
    lib().w4o_quantize_pack(_ptr(W), rows, K, group, _ptr(Wq), _ptr(S))
    return Wq, S


def dequant(Wq: np.ndarray, S: np.ndarray, group: int = 32) -> np.ndarray:
    Wq = np.ascontiguousarray(Wq, dtype=np.int32)
    S = _u16(S)
    rows, K = Wq.shape[0], Wq.shape[1] * 8
    Wdq = np.empty((rows, K), np.uint16)
    lib().w4o_dequant(_ptr(Wq), _ptr(S), rows, K, group, _ptr(Wdq))
    return Wdq


# ---- asymmetric (zero-point) quantization ---------------------------------

def quantize_zp(W: np.ndarray, group: int = 32):
    """(q uint8 [rows, K] in [0, 15], S bf16-bits [rows, K/group], Z uint8 [rows, K/group])."""
    W = _u16(W)
    rows, K = W.shape
    q = np.empty((rows, K), np.uint8)
    S = np.empty((rows, K // group), np.uint16)
    Z = np.empty((rows, K // group), np.uint8)
    lib().w4o_quantize_zp(_ptr(W), rows, K, group, _ptr(q), _ptr(S), _ptr(Z))
    return q, S, Z


def pack_u(q: np.ndarray) -> np.ndarray:
    """Unsigned codes in [0, 15] (last dim a multiple of 8) -> int32 words."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    flat = q.reshape(-1, 8)
    words = np.array([lib().w4o_pack8_u(_ptr(np.ascontiguousarray(r))) for r in flat], np.int32)
    return words.reshape(q.shape[:-1] + (q.shape[-1] // 8,))


def unpack_u(words: np.ndarray) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.int32)
    out = np.empty(words.size * 8, np.uint8)
    for j, w in enumerate(words.reshape(-1)):
        buf = np.empty(8, np.uint8)
        lib().w4o_unpack8_u(ctypes.c_int32(int(w)), _ptr(buf))
        out[8 * j:8 * j + 8] = buf
    return out.reshape(words.shape[:-1] + (words.shape[-1] * 8,))


def quantize_pack_zp(W: np.ndarray, group: int = 32):
    """(Wq int32 [rows, K/8], S bf16-bits [rows, K/group], Z uint8 [rows, K/group])."""
    W = _u16(W)
    rows, K = W.shape
    Wq = np.empty((rows, K // 8), np.int32)
    S = np.empty((rows, K // group), np.uint16)
    Z = np.empty((rows, K // group), np.uint8)
    lib().w4o_quantize_pack_zp(_ptr(W), rows, K, group, _ptr(Wq), _ptr(S), _ptr(Z))
    return Wq, S, Z


def dequant_zp(Wq: np.ndarray, S: np.ndarray, Z: np.ndarray, group: int = 32) -> np.ndarray:
    Wq = np.ascontiguousarray(Wq, dtype=np.int32)
    S = _u16(S)
    Z = np.ascontiguousarray(Z, dtype=np.uint8)
    rows, K = Wq.shape[0], Wq.shape[1] * 8
    Wdq = np.empty((rows, K), np.uint16)
    lib().w4o_dequant_zp(_ptr(Wq), _ptr(S), _ptr(Z), rows, K, group, _ptr(Wdq))
    return Wdq


def w4a16_gemm_zp(X: np.ndarray, Wq: np.ndarray, S: np.ndarray, Z: np.ndarray,
                  group: int = 32, want_r: bool = True):
    """Y = X · dequant_zp(Wq, S, Z)^T, by the plain GEMM definition."""
    return gemm(X, dequant_zp(Wq, S, Z, group), want_r)


# ---- micro-scaled FP4 (MXFP4: 32 per E8M0 scale; NVFP4: 16 per E4M3 scale) ---

def e2m1_value(code: int) -> float:
    return float(lib().w4o_e2m1_value(code))


def e2m1_encode(v: float) -> int:
    return int(lib().w4o_e2m1_encode(float(v)))


def e4m3_value(code: int) -> float:
    return float(lib().w4o_e4m3_value(code))


def e4m3_encode(v: float) -> int:
    return int(lib().w4o_e4m3_encode(float(v)))


def quantize_mxfp4(W: np.ndarray):
    """(q uint8 E2M1 codes [rows, K], E uint8 biased exponents [rows, K/32])."""
    W = _u16(W)
    rows, K = W.shape
    q = np.empty((rows, K), np.uint8)
    E = np.empty((rows, K // 32), np.uint8)
    lib().w4o_quantize_mxfp4(_ptr(W), rows, K, _ptr(q), _ptr(E))
    return q, E


def dequant_mxfp4(q: np.ndarray, E: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    E = np.ascontiguousarray(E, dtype=np.uint8)
    rows, K = q.shape
    Wdq = np.empty((rows, K), np.uint16)
    lib().w4o_dequant_mxfp4(_ptr(q), _ptr(E), rows, K, _ptr(Wdq))
    return Wdq


def quantize_nvfp4(W: np.ndarray):
    """(q uint8 E2M1 codes [rows, K], S uint8 E4M3 scales [rows, K/16], g float)."""
    W = _u16(W)
    rows, K = W.shape
    q = np.empty((rows, K), np.uint8)
    S = np.empty((rows, K // 16), np.uint8)
    g = np.zeros(1, np.float32)
    lib().w4o_quantize_nvfp4(_ptr(W), rows, K, _ptr(q), _ptr(S), _ptr(g))
    return q, S, float(g[0])


def dequant_nvfp4(q: np.ndarray, S: np.ndarray, g: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    S = np.ascontiguousarray(S, dtype=np.uint8)
    rows, K = q.shape
    Wdq = np.empty((rows, K), np.uint16)
    lib().w4o_dequant_nvfp4(_ptr(q), _ptr(S), ctypes.c_float(g), rows, K, _ptr(Wdq))
    return Wdq


def symmetric_quantize_f64(x: np.ndarray, qmax: int, group: int | None = None):
    """The generic fp64 symmetric quantizer (scale not rounded): (q, s)."""
    x = np.ascontiguousarray(x, dtype=np.float64).ravel()
    n = x.size
    group = n if group is None else group
    q = np.empty(n, np.int32)
    s = np.empty((n + group - 1) // group, np.float64)
    lib().w4o_symmetric_quantize_f64(_ptr(x), n, group, qmax, _ptr(q), _ptr(s))
    return q, s


# ---- GEMMs -----------------------------------------------------------------

def gemm(X: np.ndarray, Wdq: np.ndarray, want_r: bool = True):
    """(Y bf16-bits [M, N], R float32 [M, N]) for Y = X . Wdq^T."""
    X, Wdq = _u16(X), _u16(Wdq)
    M, K = X.shape
    N = Wdq.shape[0]
    assert Wdq.shape[1] == K
    Y = np.empty((M, N), np.uint16)
    R = np.empty((M, N), np.float32) if want_r else None
    lib().w4o_gemm(_ptr(X), _ptr(Wdq), M, N, K, _ptr(Y), _ptr(R))
    return Y, R


def w4a16_gemm(X: np.ndarray, Wq: np.ndarray, S: np.ndarray, group: int = 32,
               want_r: bool = True):
    X, S = _u16(X), _u16(S)
    Wq = np.ascontiguousarray(Wq, dtype=np.int32)
    M, K = X.shape
    N = Wq.shape[0]
    assert Wq.shape[1] * 8 == K
    Y = np.empty((M, N), np.uint16)
    R = np.empty((M, N), np.float32) if want_r else None
    lib().w4o_w4a16_gemm(_ptr(X), _ptr(Wq), _ptr(S), M, N, K, group, _ptr(Y), _ptr(R))
    return Y, R


# ---- MoE -------------------------------------------------------------------

def moe_capacity(T: int, topk: int, E: int, block: int) -> int:
    """Worst-case padded length: every expert may add block-1 padding slots."""
    cap = T * topk + E * (block - 1)
    return (cap + block - 1) // block * block


def moe_align(topk_ids: np.ndarray, E: int, block: int, cap: int | None = None):
    """(sorted_ids [cap], expert_ids [cap/block], num_post_pad)."""
    topk_ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, topk = topk_ids.shape
    if cap is None:
        cap = moe_capacity(T, topk, E, block)
    sorted_ids = np.empty(cap, np.int32)
    expert_ids = np.empty(cap // block, np.int32)
    npp = np.zeros(1, np.int32)
    rc = lib().w4o_moe_align(_ptr(topk_ids), T, topk, E, block, _ptr(sorted_ids),
                             cap, _ptr(expert_ids), _ptr(npp))
    if rc != 0:
        raise ValueError("capacity too small for the padded slot list")
    return sorted_ids, expert_ids, int(npp[0])


def moe_gemm(A: np.ndarray, a_row_div: int, Wdq: np.ndarray, sorted_ids, expert_ids,
             num_post_pad: int, num_slots: int, block: int, C_init=None,
             want_r: bool = True):
    """Grouped GEMM over the aligned slots.  Wdq is [E, N, K] bf16 bits.
    Rows of C that no real slot maps to keep C_init (default zeros)."""
    A, Wdq = _u16(A), _u16(Wdq)
    E, N, K = Wdq.shape
    C = (np.zeros((num_slots, N), np.uint16) if C_init is None
         else np.array(C_init, dtype=np.uint16, copy=True))
    R = np.zeros((num_slots, N), np.float32) if want_r else None
    sorted_ids = np.ascontiguousarray(sorted_ids, dtype=np.int32)
    expert_ids = np.ascontiguousarray(expert_ids, dtype=np.int32)
    lib().w4o_moe_gemm(_ptr(A), a_row_div, _ptr(Wdq), _ptr(sorted_ids),
                       _ptr(expert_ids), num_post_pad, num_slots, block, N, K,
                       _ptr(C), _ptr(R))
    return C, R


def moe_gate_topk(logits: np.ndarray, topk: int):
    """Router gating: (topk_ids int32 [T, topk], topk_weights float32 [T, topk]).
    p = softmax(logits) per token in fp32; the topk largest p in descending
    order, ties to the lower expert id (decided on the logits: the order of the
    exact p); weights = the selected p, not renormalized."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, topk), np.int32)
    w = np.empty((T, topk), np.float32)
    lib().w4o_moe_gate_topk(_ptr(logits), T, E, topk, _ptr(ids), _ptr(w))
    return ids, w


def moe_combine(D: np.ndarray, w: np.ndarray, topk: int) -> np.ndarray:
    """out[t, n] = bf16(sum_k w[t, k] * D[t*topk + k, n]), fp32, ascending k."""
    D = _u16(D)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T = w.shape[0]
    N = D.shape[1]
    out = np.empty((T, N), np.uint16)
    lib().w4o_moe_combine(_ptr(D), _ptr(w), T, topk, N, _ptr(out))
    return out


def silu_mul(gate_up: np.ndarray) -> np.ndarray:
    """MoE glue between the two grouped GEMMs (not a graded kernel):
    h = bf16(silu(g) * u) with g the first half of the columns and u the second,
    silu(x) = x / (1 + exp(-x)) in fp32."""
    gu = bf16_to_f32(_u16(gate_up))
    half = gu.shape[1] // 2
    g, u = gu[:, :half].astype(np.float32), gu[:, half:].astype(np.float32)
    h = (g / (np.float32(1.0) + np.exp(-g))) * u
    return f32_to_bf16_bits(h.astype(np.float32))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (ties to even), returned as raw bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    upper = (u >> 16).astype(np.uint32)
    lower = u & np.uint32(0xFFFF)
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + round_up.astype(np.uint32)).astype(np.uint16)
