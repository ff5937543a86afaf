"""The allocation-free GEMM entry point, called through the C ABI.

w4a16_gemm_noalloc exists for callers that cannot give the library a device
workspace (an engine that fixes its device memory budget at start-up, a
plug-in whose host framework owns the allocator, code that must not call
cudaMalloc).  It must give the same product as w4a16_gemm with a workspace, call
after call, while using only the library's own fixed scratch array.  This file
is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits

pytestmark = pytest.mark.gpu
REL_TOL = 1e-2


def _close_to_oracle(y_bits, R, what):
    y = (y_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = R.astype(np.float64)
    scale = np.abs(r).max()
    err = np.abs(y - r)
    assert err.max() <= REL_TOL * scale, what
    assert not np.any(err > REL_TOL * np.abs(r) + 1e-3 * scale), what


@pytest.mark.parametrize("M,N", [(1, 12288), (16, 12288), (32, 12288), (48, 4096)])
def test_noalloc_matches_workspace_entry_point_twice(M, N):
    """Two calls in a row give the very bits of w4a16_gemm with a caller
    workspace: both run the same schedule and add the split's partial sums in
    the same fixed order, so a wrongly zeroed counter in the shared array would
    show as a difference.  M = 16, 32 and 48 run the split (scratch in use;
    ~6 MB of the 8 MiB array for M = 48 on 4096 weight rows); M = 1 the
    warp-level kernel, which needs none.  M > 1 is also checked against the
    oracle's FP32-accumulated product."""
    L = w4.lib()
    cfg = synth.Decode()
    Wq_h, S_h = _decode_weight()
    Wq_h, S_h = np.ascontiguousarray(Wq_h[:N]), np.ascontiguousarray(S_h[:N])
    dev = "cuda"
    Wq = torch.from_numpy(Wq_h).to(dev)
    S = torch.from_numpy(S_h.view(np.int16)).view(torch.bfloat16).to(dev)
    X = cfg.activations(M, dev)
    K = cfg.K
    stream = torch.cuda.current_stream().cuda_stream
    need = L.w4a16_gemm_workspace_bytes(M, N, K)
    assert (need > 0) == (M > 8), "the split schedule (scratch) is what M > 8 exercises"
    assert need <= (8 << 20)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    rc = L.w4a16_gemm(X.data_ptr(), Wq.data_ptr(), S.data_ptr(), Y_ref.data_ptr(), M, N, K, 32,
                      ws.data_ptr(), ws.numel(), stream)
    assert rc == 0
    for call in range(2):                       # two calls in a row share the array
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        rc = L.w4a16_gemm_noalloc(X.data_ptr(), Wq.data_ptr(), S.data_ptr(), Y.data_ptr(),
                                  M, N, K, 32, stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        assert np.array_equal(bits(Y), bits(Y_ref)), f"M={M} call {call}: not the same bits"
    assert L.w4_device_status(stream) == 0
    if M > 1:
        _, R = oracle.w4a16_gemm(bits(X), Wq_h, S_h)
        _close_to_oracle(bits(Y), R, f"M={M} against the oracle")


_DECODE = {}


def _decode_weight():
    if "w" not in _DECODE:
        _DECODE["w"] = oracle.quantize_pack(bits(synth.Decode().weight()))
    return _DECODE["w"]


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = w4.lib()
    cfg = synth.Decode()
    M, N, K = 64, cfg.N, cfg.K                  # split scratch ~9.4 MB > 8 MiB
    assert L.w4a16_gemm_workspace_bytes(M, N, K) > (8 << 20)
    dev = "cuda"
    X = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    Wq = torch.zeros((N, K // 8), dtype=torch.int32, device=dev)
    S = torch.zeros((N, K // 32), dtype=torch.bfloat16, device=dev)
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device=dev)
    rc = L.w4a16_gemm_noalloc(X.data_ptr(), Wq.data_ptr(), S.data_ptr(), Y.data_ptr(), M, N, K,
                              32, torch.cuda.current_stream().cuda_stream)
    assert rc == 2                              # W4_ERR_UNSUPPORTED, nothing launched
