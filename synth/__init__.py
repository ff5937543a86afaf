"""Seeded synthetic inputs for the INT4 W4A16 hot path.

Shared by the tests (both the CUDA path and the CPU oracle receive the very same
tensors) and by ``bench.py``.  This module holds input generation only: random
draws, casts to BF16 and the workload shapes.  It contains none of the method's
arithmetic (no scale, rounding, packing, GEMM or alignment).

Recipes:
  * values are drawn in fp32 and cast to BF16 with round-to-nearest-even
    (``Tensor.to(torch.bfloat16)``);
  * every tensor has its own generator seeded with ``seed * 1000 + index``;
  * "0.1 % entries x20 outliers": exactly ``round(0.001 * numel)`` distinct
    positions drawn uniformly without replacement, multiplied by 20 in fp32
    before the BF16 cast;
  * Laplace(0, b) is drawn by inverse CDF from a uniform draw, scale b;
  * MoE routing: logits ~ N(0, 1) fp32, softmax in fp32, top-k by probability
    with ties going to the lower expert id, weights are the selected
    probabilities (not renormalized).

Draws on a CUDA device use CUDA generators and therefore differ bitwise from
CPU draws with the same seed; callers that need the oracle to see the same
input copy the generated tensor to the host.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _gen(seed: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(index))
    return g


def normal_bf16(shape, std: float, seed: int, index: int = 0, device="cpu",
                outlier_frac: float = 0.0, outlier_mult: float = 20.0) -> torch.Tensor:
    """N(0, std^2) BF16 tensor, optionally with a fraction of entries scaled."""
    g = _gen(seed, index, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(std)
    if outlier_frac > 0.0:
        n = x.numel()
        count = int(round(outlier_frac * n))
        if count > 0:
            pos = torch.randperm(n, generator=g, device=device)[:count]
            flat = x.view(-1)
            flat[pos] = flat[pos] * outlier_mult
    return x.to(torch.bfloat16)


def laplace_bf16(shape, b: float, seed: int, index: int = 0, device="cpu") -> torch.Tensor:
    """Laplace(0, b) BF16 tensor (location 0, scale b), by inverse CDF."""
    g = _gen(seed, index, device)
    # u in [-0.5 + 2^-25, 0.5): strictly inside (-1/2, 1/2), so 1 - 2|u| > 0 and
    # every draw is finite (a draw of exactly -1/2 would map to infinity).
    u = (torch.rand(shape, generator=g, device=device, dtype=torch.float32) - 0.5) \
        * (1.0 - 2.0 ** -24)
    x = -b * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    return x.to(torch.bfloat16)


def router_logits(T: int, E: int, seed: int, index: int = 0, device="cpu"):
    """Router logits ~ N(0, 1), float32 [T, E] (the input of the gating kernel)."""
    g = _gen(seed, index, "cpu")
    return torch.randn((T, E), generator=g, dtype=torch.float32).to(device)


def routing(T: int, E: int, topk: int, seed: int, index: int = 0, skew: float = 0.0):
    """Router logits ~ N(0,1) [T, E] -> softmax -> top-k (ties to lower id).
    skew > 0 adds -skew * log(1 + e) to expert e's logit (a Zipf-like load: the
    low ids are hot).  Returns (topk_ids int32 [T, topk], topk_weights float32
    [T, topk]) on CPU."""
    g = _gen(seed, index, "cpu")
    logits = torch.randn((T, E), generator=g, dtype=torch.float32)
    if skew:
        logits = logits - skew * torch.log1p(torch.arange(E, dtype=torch.float32))
    p = torch.softmax(logits, dim=-1)
    order = torch.argsort(-p, dim=-1, stable=True)[:, :topk]
    w = torch.gather(p, 1, order)
    return order.to(torch.int32).contiguous(), w.contiguous()


# ---------------------------------------------------------------------------
# Workload shapes
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class TinyLayer:
    """Single layer: W[1024, 1024] ~ N(0, 0.02^2), X[4, 1024] ~ N(0, 1), seed 0."""
    N: int = 1024
    K: int = 1024
    M: int = 4
    seed: int = 0

    def weight(self, device="cpu"):
        return normal_bf16((self.N, self.K), 0.02, self.seed, 0, device)

    def activations(self, device="cpu"):
        return normal_bf16((self.M, self.K), 1.0, self.seed, 1, device)


@dataclass(frozen=True)
class Decode:
    """Decode GEMV sweep: W[12288, 4096] ~ N(0, 0.02^2) with 0.1 % x20 outliers,
    X[M, 4096] ~ N(0, 1) for M in {1, 8, 16, 32}."""
    N: int = 12288
    K: int = 4096
    Ms: tuple = (1, 8, 16, 32)
    seed: int = 0

    def weight(self, device="cpu"):
        return normal_bf16((self.N, self.K), 0.02, self.seed, 0, device,
                           outlier_frac=0.001, outlier_mult=20.0)

    def activations(self, M: int, device="cpu"):
        return normal_bf16((M, self.K), 1.0, self.seed, 10 + M, device)

    def grads(self, device="cpu"):
        """BF16 gradients of the fake-quantized weight, ~ N(0, 1e-3^2)."""
        return normal_bf16((self.N, self.K), 1e-3, self.seed, 5, device)


@dataclass(frozen=True)
class Prefill:
    """Prefill GEMM: W[18432, 7168] ~ Laplace(0, 0.015), X[M, 7168] ~ N(0, 1),
    M in {512, 2048, 8192}."""
    N: int = 18432
    K: int = 7168
    Ms: tuple = (512, 2048, 8192)
    seed: int = 0

    def weight(self, device="cpu"):
        return laplace_bf16((self.N, self.K), 0.015, self.seed, 0, device)

    def activations(self, M: int, device="cpu"):
        return normal_bf16((M, self.K), 1.0, self.seed, 10 + M % 997, device)


@dataclass(frozen=True)
class MoEDecode:
    """MoE decode layer: 128 experts, top-8, hidden 4096, intermediate 1536;
    gate_up W[3072, 4096] and down W[4096, 1536] per expert ~ N(0, 0.02^2);
    T tokens in {16, 64, 256}; block in {16, 32, 64}."""
    E: int = 128
    topk: int = 8
    hidden: int = 4096
    inter: int = 1536
    Ts: tuple = (16, 64, 256)
    blocks: tuple = (16, 32, 64)
    seed: int = 0

    def gate_up_weight(self, device="cpu"):
        return normal_bf16((self.E, 2 * self.inter, self.hidden), 0.02, self.seed, 0, device)

    def down_weight(self, device="cpu"):
        return normal_bf16((self.E, self.hidden, self.inter), 0.02, self.seed, 1, device)

    def tokens(self, T: int, device="cpu"):
        return normal_bf16((T, self.hidden), 1.0, self.seed, 100 + T, device)

    def routing(self, T: int, skew: float = 0.0):
        return routing(T, self.E, self.topk, self.seed, 200 + T, skew)

    def logits(self, T: int, device="cpu"):
        return router_logits(T, self.E, self.seed, 200 + T, device)


@dataclass(frozen=True)
class QATStack:
    """QAT weight pass over a 48-layer stack: each layer holds W[12288, 4096] and
    W[4096, 12288] ~ N(0, 0.02^2) with 0.1 % x20 outliers; grads ~ N(0, 1e-3^2)."""
    layers: int = 48
    shapes: tuple = ((12288, 4096), (4096, 12288))
    seed: int = 0

    def weight(self, layer: int, which: int, device="cpu"):
        return normal_bf16(self.shapes[which], 0.02, self.seed, 1000 + 2 * layer + which,
                           device, outlier_frac=0.001, outlier_mult=20.0)

    def grad(self, layer: int, which: int, device="cpu"):
        return normal_bf16(self.shapes[which], 1e-3, self.seed, 5000 + 2 * layer + which, device)

    @property
    def elements(self) -> int:
        return self.layers * sum(r * c for r, c in self.shapes)


def bits(t: torch.Tensor):
    """Raw BF16 bit patterns of a (CPU or CUDA) BF16 tensor, as a numpy uint16 array."""
    import numpy as np
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
