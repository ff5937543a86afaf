"""Bounded device waits: a wait that runs out is reported on the host and leaves
the CUDA context usable (failure detection without a GPU fault)."""
import numpy as np
import pytest
import torch

import int4_w4a16_b200 as w4
import oracle
import synth
from synth import bits

pytestmark = pytest.mark.gpu

W4_ERR_TIMEOUT = 4


def test_wait_runs_out_and_reports_timeout():
    w4.w4_device_status()                       # clean slate
    w4.w4_wait_selftest(20000)                  # 20 ms limit on a phase nothing completes
    with pytest.raises(w4.W4Error) as e:
        w4.w4_device_status()
    assert e.value.code == W4_ERR_TIMEOUT
    w4.w4_device_status()                       # the flag was cleared by the report

    # the context is still usable: a small quantize + GEMM matches the oracle
    W = synth.normal_bf16((256, 512), 0.02, seed=5)
    X = synth.normal_bf16((4, 512), 1.0, seed=6)
    Wq_o, S_o = oracle.quantize_pack(bits(W))
    Wq, S = w4.quantize_pack(W.cuda())
    Y = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    w4.w4a16_gemm(X.cuda(), Wq, S, Y)
    w4.w4_device_status()
    assert np.array_equal(Wq.cpu().numpy(), Wq_o)
    _, R = oracle.w4a16_gemm(bits(X), Wq_o, S_o)
    R = R.astype(np.float64)
    y = (bits(Y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.abs(y - R).max() <= 1e-2 * np.abs(R).max()
