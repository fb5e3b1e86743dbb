"""Seeded synthetic workloads for the QLoRA NF4 linear layer.

This module only draws random inputs; it holds none of the method's arithmetic,
so both the CUDA path and the CPU oracle can be fed from it.  Every tensor is
drawn on the host from a ``torch.Generator`` seeded per workload and per
projection: the weights (W, then A, then B) come from one generator that does
not depend on the token count, so decode runs with 1, 4 or 16 tokens share one
quantized weight; the activations (X, then dY) come from a second generator
seeded with the token count.

Shapes and distributions follow the five workloads the layer is measured on:

* ``fwd_2048``       one linear, forward only: X [128, 2048] ~ N(0,1) bf16,
                     W 2048x2048 ~ N(0, 0.02), r = 8, alpha = 16,
                     A ~ U(+-1/sqrt 2048), B ~ N(0, 0.01).
* ``qproj_7b``       Llama-7B-shaped q_proj, forward and backward: X [4096 (4x1024
                     tokens), 4096], dY ~ N(0,1), W 4096x4096 ~ N(0, 0.02), r = 16,
                     alpha = 32, A ~ U(+-1/64), B ~ N(0, 0.01).
* ``mlp_7b``         gate/up 4096 -> 11008 and down 11008 -> 4096, 8192 tokens,
                     r = 64, alpha = 128 (A ~ U(+-1/sqrt K), B ~ N(0, 0.01): the same
                     recipe as the two workloads above, which give it explicitly).
* ``decode_70b_up``  W 8192 -> 28672 ~ N(0, 0.02) with 1 % of entries (uniform
                     seeded choice) set to +-6 sigma with a random sign; 1, 4 or 16
                     tokens; r = 16, alpha = 32; forward only.
* ``layer_70b``      all 7 projections of a 70B-shaped decoder layer (q, o 8192x8192;
                     k, v 1024x8192; gate, up 28672x8192; down 8192x28672), 4096
                     tokens, r = 64, alpha = 16.

Weight shapes are ``[N, K]`` = [out_features, in_features] (the nn.Linear layout);
LoRA A is ``[r, K]`` and B is ``[N, r]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Projection:
    name: str
    N: int  # out features
    K: int  # in features


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    M: int
    r: int
    alpha: float
    projections: tuple
    backward: bool
    a_bound: str = "1/sqrt(K)"  # U(-b, b) for A
    b_std: float = 0.01
    w_std: float = 0.02
    outlier_frac: float = 0.0
    outlier_sigmas: float = 6.0
    m_list: tuple = field(default_factory=tuple)  # decode token counts

    @property
    def scale(self) -> float:
        return self.alpha / self.r


WORKLOADS = {
    "fwd_2048": Workload("fwd_2048", 0, 128, 8, 16.0, (Projection("linear", 2048, 2048),), False),
    "qproj_7b": Workload("qproj_7b", 1, 4096, 16, 32.0, (Projection("q_proj", 4096, 4096),), True),
    "mlp_7b": Workload("mlp_7b", 2, 8192, 64, 128.0,
                       (Projection("gate_proj", 11008, 4096), Projection("up_proj", 11008, 4096),
                        Projection("down_proj", 4096, 11008)), True),
    "decode_70b_up": Workload("decode_70b_up", 3, 16, 16, 32.0, (Projection("up_proj", 28672, 8192),),
                              False, outlier_frac=0.01, m_list=(1, 4, 16)),
    "layer_70b": Workload("layer_70b", 4, 4096, 64, 16.0,
                          (Projection("q_proj", 8192, 8192), Projection("k_proj", 1024, 8192),
                           Projection("v_proj", 1024, 8192), Projection("o_proj", 8192, 8192),
                           Projection("gate_proj", 28672, 8192), Projection("up_proj", 28672, 8192),
                           Projection("down_proj", 8192, 28672)), True),
}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def draw_weight(g: torch.Generator, N: int, K: int, std: float, outlier_frac: float = 0.0,
                outlier_sigmas: float = 6.0) -> torch.Tensor:
    """fp32 [N, K] ~ N(0, std); optionally a seeded uniform fraction of entries
    replaced by +-outlier_sigmas*std with a random sign."""
    W = torch.randn(N, K, generator=g, dtype=torch.float32) * std
    if outlier_frac > 0:
        pick = torch.rand(N, K, generator=g) < outlier_frac
        sign = torch.randint(0, 2, (N, K), generator=g, dtype=torch.int8).to(torch.float32) * 2 - 1
        W = torch.where(pick, sign * (outlier_sigmas * std), W)
    return W


def draw_linear(wl: Workload, proj_index: int = 0, M: int | None = None, with_dy: bool | None = None,
                with_x: bool = True):
    """Inputs of one projection of a workload, all on the host.

    Returns a dict with X (bf16 [M,K]), W (fp32 [N,K]), A (bf16 [r,K]),
    B (bf16 [N,r]), dY (bf16 [M,N], when the workload has a backward pass),
    scale (alpha / r) and the shapes."""
    p = wl.projections[proj_index]
    M = wl.M if M is None else int(M)
    with_dy = wl.backward if with_dy is None else with_dy
    gw = generator(wl.seed * 1000 + proj_index)
    gx = generator(wl.seed * 1000 + 500 + proj_index * 37 + M)
    out = {"M": M, "N": p.N, "K": p.K, "r": wl.r, "scale": wl.scale, "name": p.name}
    out["W"] = draw_weight(gw, p.N, p.K, wl.w_std, wl.outlier_frac, wl.outlier_sigmas)
    bound = 1.0 / math.sqrt(p.K)
    out["A"] = ((torch.rand(wl.r, p.K, generator=gw, dtype=torch.float32) * 2 - 1) * bound).to(torch.bfloat16)
    out["B"] = (torch.randn(p.N, wl.r, generator=gw, dtype=torch.float32) * wl.b_std).to(torch.bfloat16)
    out["X"] = torch.randn(M, p.K, generator=gx, dtype=torch.float32).to(torch.bfloat16) if with_x else None
    if with_dy:
        out["dY"] = torch.randn(M, p.N, generator=gx, dtype=torch.float32).to(torch.bfloat16)
    return out


def draw_small(seed: int, M: int, N: int, K: int, r: int, alpha: float, w_std: float = 0.02,
               b_std: float = 0.01, with_dy: bool = True):
    """A small ad-hoc problem with the same recipe (for ragged/edge tests)."""
    g = generator(seed)
    X = torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g, dtype=torch.float32) * w_std
    bound = 1.0 / math.sqrt(K)
    A = ((torch.rand(r, K, generator=g) * 2 - 1) * bound).to(torch.bfloat16)
    B = (torch.randn(N, r, generator=g) * b_std).to(torch.bfloat16)
    out = {"M": M, "N": N, "K": K, "r": r, "scale": alpha / r, "X": X, "W": W, "A": A, "B": B}
    if with_dy:
        out["dY"] = torch.randn(M, N, generator=g).to(torch.bfloat16)
    return out


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bits of a bf16 tensor as a numpy array (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
