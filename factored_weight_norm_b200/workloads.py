"""Seeded synthetic inputs for the DoRA factored-norm / compose path.

This module only draws random tensors with the shapes, scales and value
distributions of the workloads below.  It holds none of the method's
arithmetic (no norm of W + sBA, no compose); the CUDA library and the CPU
oracle both consume what it produces.  Random draws happen in a fixed order
(W, A, B, magnitude noise, x, dy) from one ``torch.Generator`` seeded per
workload, so a (workload, device) pair always yields the same tensors.

Workload shapes follow the problem the pages describe ("Scaling DoRA:
High-Rank Adaptation via Factored Norms and Fused Kernels", Abstract:
d_in = 8192 at rank r = 384 in bf16, adapters on 8-32B models): a tiny fp32
module, a 4096^2 r=64 module, the 8192^2 r=384 headline module, the MLP
up-projection of a ~32B decoder (5120 -> 27648), and rank / token sweeps.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "RANK_SWEEP",
    "TOKEN_SWEEP",
    "headline",
    "make_weights",
    "make_activations",
    "make_grad",
    "make_near_unity_mn",
    "torch_dtype",
]


@dataclass(frozen=True)
class Workload:
    """One adapted linear module plus a batch of tokens.

    ``w_std``/``b_std`` are the standard deviations of W and B (normal);
    A is uniform on +-1/sqrt(d_in); ``m_noise`` is the relative spread of the
    magnitude around the base row norm (m = ||W_i|| * (1 + N(0, m_noise))).
    """

    name: str
    d_out: int
    d_in: int
    r: int
    s: float
    tokens: int
    dtype: str = "bf16"  # "bf16" or "f32": type of W, A, B and activations
    w_std: float = 0.015
    b_std: float = 0.002
    m_noise: float = 5e-4
    seed: int = 1234

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny_f32", 64, 128, 8, 2.0, 32, "f32", 0.02, 0.01, 1e-3, 1235)
SINGLE_4096 = Workload("bf16_4096_r64", 4096, 4096, 64, 2.0, 4096, "bf16", 0.02, 0.005, 1e-3, 1236)
HEADLINE = Workload("bf16_8192_r384", 8192, 8192, 384, 0.5, 8192, "bf16", 0.015, 0.002, 5e-4, 1237)
MLP_UP_32B = Workload("bf16_mlp_up_5120x27648_r384", 27648, 5120, 384, 0.5, 16384, "bf16", 0.01, 0.002, 5e-4, 1238)

WORKLOADS = {w.name: w for w in (TINY_F32, SINGLE_4096, HEADLINE, MLP_UP_32B)}

# rank sweep at d_out = d_in = 8192 with the headline generators
RANK_SWEEP = tuple(
    HEADLINE.with_(name=f"bf16_8192_r{r}", r=r, seed=1239) for r in (16, 64, 128, 256, 384, 512, 768)
)
# compose-only sweep over tokens at d_out = 8192 (g = 1 + N(0, 1e-4))
TOKEN_SWEEP = tuple(
    HEADLINE.with_(name=f"compose_T{t}", tokens=t, seed=1239) for t in (1024, 4096, 16384, 65536)
)


def headline() -> Workload:
    return HEADLINE


def torch_dtype(wl: Workload) -> torch.dtype:
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def _gen(wl: Workload, device, salt: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 1000 + salt)
    return g


def make_weights(wl: Workload, device="cpu"):
    """W [d_out, d_in], A [r, d_in], B [d_out, r] in the workload dtype, m fp32 [d_out].

    m is drawn around the base row norm so that m / ||W + sBA|| sits in the
    near-unity regime the Scaling DoRA abstract describes.
    """
    dt = torch_dtype(wl)
    g = _gen(wl, device, 1)
    W = (torch.randn(wl.d_out, wl.d_in, generator=g, device=device) * wl.w_std).to(dt)
    bound = 1.0 / math.sqrt(wl.d_in)
    A = ((torch.rand(wl.r, wl.d_in, generator=g, device=device) * 2.0 - 1.0) * bound).to(dt)
    B = (torch.randn(wl.d_out, wl.r, generator=g, device=device) * wl.b_std).to(dt)
    noise = torch.randn(wl.d_out, generator=g, device=device) * wl.m_noise
    base_scale = torch.linalg.vector_norm(W.float(), dim=1)
    m = (base_scale * (1.0 + noise)).float()
    return W, A, B, m


def make_activations(wl: Workload, W, A, B, device="cpu", tokens=None):
    """x ~ N(0, 1) [tokens, d_in]; base = x W^T and lora = (x A^T) B^T, [tokens, d_out].

    These are inputs of the compose step; they are produced with ordinary
    matmuls on ``device`` and handed unchanged to both the library and the
    oracle.
    """
    dt = torch_dtype(wl)
    T = wl.tokens if tokens is None else tokens
    g = _gen(wl, device, 2)
    x = torch.randn(T, wl.d_in, generator=g, device=device).to(dt)
    if T == 0:
        empty = torch.empty(0, wl.d_out, dtype=dt, device=device)
        return x, empty, empty.clone()
    base = x @ W.t()
    lora = (x @ A.t()) @ B.t()
    return x, base.to(dt).contiguous(), lora.to(dt).contiguous()


def make_grad(wl: Workload, device="cpu", tokens=None):
    """Upstream gradient dy ~ N(0, 1) [tokens, d_out] in the workload dtype."""
    T = wl.tokens if tokens is None else tokens
    g = _gen(wl, device, 3)
    return torch.randn(T, wl.d_out, generator=g, device=device).to(torch_dtype(wl))


def make_near_unity_mn(wl: Workload, W, device="cpu", spread=1e-4):
    """(m, n) fp32 with m = ||W_i|| and n = m / (1 + N(0, spread)).

    Used by compose-only cases, where n is an input rather than the output of
    the norm, so that g = m / n - 1 is of order ``spread``.
    """
    g = _gen(wl, device, 4)
    m = torch.linalg.vector_norm(W.float(), dim=1).float()
    gg = 1.0 + torch.randn(wl.d_out, generator=g, device=device) * spread
    n = (m / gg).float()
    return m, n
