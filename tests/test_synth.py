"""The seeded input generators produce what the workload recipes state."""
import torch

import synth


def test_generators_finite_and_shaped():
    for t in [synth.normal_bf16((64, 4096), 0.02, 0, outlier_frac=0.001),
              synth.laplace_bf16((1024, 7168), 0.015, 0),
              synth.Prefill().weight()[:2048]]:
        assert t.dtype == torch.bfloat16
        assert torch.isfinite(t.float()).all()


def test_outlier_count_and_laplace_scale():
    base = synth.normal_bf16((1000, 1000), 0.02, 3)
    out = synth.normal_bf16((1000, 1000), 0.02, 3, outlier_frac=0.001)
    assert int((base != out).sum()) <= 1000
    assert int((out.float().abs() > 0.2).sum()) > 300        # x20 of N(0, 0.02)
    lap = synth.laplace_bf16((4096, 1024), 0.015, 1).float()
    assert abs(lap.abs().mean().item() - 0.015) < 3e-4         # E|x| = b


def test_routing_topk_properties():
    ids, w = synth.routing(64, 128, 8, seed=5)
    assert ids.shape == (64, 8) and ids.dtype == torch.int32
    assert all(len(set(r.tolist())) == 8 for r in ids)
    assert torch.all(w[:, :-1] >= w[:, 1:])                   # descending probability
    assert torch.all(w.sum(1) < 1.0)                          # not renormalized


def test_seeded_determinism():
    a = synth.Decode().activations(8)
    b = synth.Decode().activations(8)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
