"""Seeded synthetic inputs for the rotated quantized linear layer.

This module only draws random numbers; it holds none of the method's arithmetic
and is shared by the CUDA path's tests/benchmark and by the oracle's tests.

Distributions (Llama shapes only; no weights or datasets are involved):
  * activations X ~ N(0, 1) in fp32, with a fixed seeded set of outlier
    channels (columns) multiplied by 50, then rounded to bf16.  The outlier
    set is ``randperm(K, seed 1234)[:n]`` with n = max(4, round(0.001 K)),
    i.e. 4, 8, 11 and 29 channels for K = 4096, 8192, 11008 and 28672.
  * weights W ~ N(0, 0.02^2), bf16.
  * output gradients dY ~ N(0, 1e-3^2), bf16.
Every tensor is drawn in fp32 from a ``torch.Generator`` on the target device,
seeded per tensor, then cast to bf16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

OUTLIER_SCALE = 50.0
WEIGHT_SIGMA = 0.02
GRAD_SIGMA = 1e-3


def outlier_channels(k: int) -> torch.Tensor:
    n = max(4, int(round(0.001 * k)))
    g = torch.Generator().manual_seed(1234)
    return torch.randperm(k, generator=g)[:n]


def _normal(rows: int, cols: int, seed: int, device, sigma: float) -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(int(seed))
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x


def activations(rows: int, cols: int, seed: int, device="cpu", outliers: bool = True) -> torch.Tensor:
    x = _normal(rows, cols, seed, device, 1.0)
    if outliers:
        idx = outlier_channels(cols).to(x.device)
        x[:, idx] *= OUTLIER_SCALE
    return x.to(torch.bfloat16)


def weights(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    return _normal(rows, cols, seed, device, WEIGHT_SIGMA).to(torch.bfloat16)


def grads(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    return _normal(rows, cols, seed, device, GRAD_SIGMA).to(torch.bfloat16)


def plain(rows: int, cols: int, seed: int, device="cpu", sigma: float = 1.0) -> torch.Tensor:
    """N(0, sigma^2) bf16 with no outlier channels."""
    return _normal(rows, cols, seed, device, sigma).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# Workload definitions (sizes of the five Llama-shaped cases).
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class Gemm:
    """One linear layer of a transformer block: X[M,K] @ W[N,K]^T."""

    name: str
    m: int  # tokens
    n: int  # output features
    k: int  # input features
    x_key: str  # which activation tensor feeds it (shared across q/k/v and gate/up)


@dataclass
class LayerShapes:
    tokens: int = 4096
    hidden: int = 8192
    ffn: int = 28672
    kv: int = 1024  # 8 KV heads of 128 (grouped-query attention)
    gemms: list = field(default_factory=list)

    def __post_init__(self):
        if self.gemms:
            return  # an explicit GEMM list (a single-GEMM case)
        t, h, f, kv = self.tokens, self.hidden, self.ffn, self.kv
        self.gemms = [
            Gemm("q", t, h, h, "attn_in"),
            Gemm("k", t, kv, h, "attn_in"),
            Gemm("v", t, kv, h, "attn_in"),
            Gemm("o", t, h, h, "attn_out"),
            Gemm("gate", t, f, h, "mlp_in"),
            Gemm("up", t, f, h, "mlp_in"),
            Gemm("down", t, h, f, "mlp_act"),
        ]

    def total_ops(self, kinds=("fwd", "dx", "dw")) -> int:
        """2 * M * N * K summed over the GEMMs of the listed kinds (forward, dX, dW
        each multiply the same three sizes)."""
        return sum(len(kinds) * 2 * g.m * g.n * g.k for g in self.gemms)


LLAMA70B_LAYER = LayerShapes()
# Single-GEMM Llama-7B cases: the attention projection forward (X[8192,4096],
# W[4096,4096]) and the FFN down-projection backward (dY[8192,4096],
# W[4096,11008], X[8192,11008]).
LLAMA7B_ATTN_PROJ = LayerShapes(tokens=8192, hidden=4096, ffn=11008, kv=4096,
                                gemms=[Gemm("proj", 8192, 4096, 4096, "attn_in")])
LLAMA7B_FFN_DOWN = LayerShapes(tokens=8192, hidden=4096, ffn=11008, kv=4096,
                               gemms=[Gemm("down", 8192, 4096, 11008, "mlp_act")])
# One GEMM of the Llama-70B layer: the gate projection (X[4096,8192], W[28672,8192]).
LLAMA70B_GATE = LayerShapes(gemms=[Gemm("gate", 4096, 28672, 8192, "mlp_in")])
# Another: the query projection (X[4096,8192], W[8192,8192]).
LLAMA70B_Q = LayerShapes(gemms=[Gemm("q", 4096, 8192, 8192, "attn_in")])


def layer_inputs(shapes: LayerShapes, seed: int, device) -> dict:
    """All tensors of one layer step: activations, weights and output gradients."""
    t = shapes.tokens
    out = {"x": {}, "w": {}, "dy": {}}
    in_dims = {}
    for g in shapes.gemms:
        in_dims[g.x_key] = g.k
    for i, (key, k) in enumerate(sorted(in_dims.items())):
        out["x"][key] = activations(t, k, seed * 1000 + 1 + i, device)
    for i, g in enumerate(shapes.gemms):
        out["w"][g.name] = weights(g.n, g.k, seed * 1000 + 100 + i, device)
        out["dy"][g.name] = grads(t, g.n, seed * 1000 + 200 + i, device)
    return out
