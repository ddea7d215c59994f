"""Seeded synthetic inputs shaped like the DiT layers the method is used on.

This module holds no arithmetic of the method: it only draws random numbers with a seeded
CPU ``torch.Generator`` and rounds them to bf16. The same bytes feed the CUDA library and
the CPU oracle.

Recipe (shapes are the DiT geometries named on the SD.Next benchmark commit log: Flux.1
attention linears 3072x3072, feed-forward 12288x3072, 4608 joint tokens):

* draw fp32 from the stated distribution, scale, then round to bf16 (round-to-nearest-even);
* "outlier channels": ``round(frac * K)`` input columns chosen by ``randperm(K)`` from the same
  generator, multiplied by the stated factor before rounding;
* Student-t(nu) is drawn as ``z / sqrt(chi2_nu / nu)`` with ``chi2_nu`` a sum of ``nu`` squared
  standard normals (nu integer), which is the textbook construction;
* draw order within a case: x, outlier columns, W (or W_up, W_down), bias, A, B;
* input-gradient cases (the backward pass through a frozen layer of N outputs and K inputs):
  dy [M, N] ~ N(0, dy_std^2) with outlier columns, then W [N, K]; dy is kept in ``x``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a CPU bf16 tensor, as a numpy uint16 array (no copy)."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """CPU bf16 tensor whose bit patterns are the given uint16 array."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _normal(gen, shape, std=1.0):
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def _student_t(gen, shape, nu: int):
    z = torch.randn(*shape, generator=gen, dtype=torch.float32)
    chi2 = torch.zeros(shape, dtype=torch.float32)
    for _ in range(nu):
        e = torch.randn(*shape, generator=gen, dtype=torch.float32)
        chi2 += e * e
    return z / torch.sqrt(chi2 / nu)


def activations(gen, M, K, dist="normal", outlier_frac=0.0, outlier_count=None,
                outlier_factor=1.0, nu=4):
    """x [M, K] bf16 with optional outlier columns."""
    if dist == "normal":
        x = _normal(gen, (M, K))
    elif dist == "student_t":
        x = _student_t(gen, (M, K), nu)
    else:
        raise ValueError(dist)
    count = outlier_count if outlier_count is not None else int(round(outlier_frac * K))
    cols = torch.randperm(K, generator=gen)[:count]
    if count:
        x[:, cols] *= outlier_factor
    return x.to(torch.bfloat16), cols


@dataclass
class Case:
    """One synthetic layer problem (all tensors CPU bf16)."""
    name: str
    M: int
    N: int
    K: int
    g: int
    x: torch.Tensor
    W: torch.Tensor
    bias: torch.Tensor | None = None
    A: torch.Tensor | None = None
    B: torch.Tensor | None = None
    lora_scale: float = 1.0
    extra: dict = field(default_factory=dict)


def make_case(M, N, K, g=256, seed=0, dist="normal", outlier_frac=0.0,
              outlier_count=None, outlier_factor=1.0, w_std=0.02, bias_std=None,
              lora_rank=0, lora_std=0.01, lora_scale=1.0, name="case") -> Case:
    gen = torch.Generator("cpu").manual_seed(seed)
    x, cols = activations(gen, M, K, dist, outlier_frac, outlier_count, outlier_factor)
    W = _normal(gen, (N, K), w_std).to(torch.bfloat16)
    bias = _normal(gen, (N,), bias_std).to(torch.bfloat16) if bias_std else None
    A = B = None
    if lora_rank:
        A = _normal(gen, (K, lora_rank), lora_std).to(torch.bfloat16)
        B = _normal(gen, (lora_rank, N), lora_std).to(torch.bfloat16)
    return Case(name, M, N, K, g, x, W, bias, A, B, lora_scale,
                extra={"outlier_cols": cols, "seed": seed})


# The five DiT-shaped workloads. Seeds are the workload's index (0..4).
WORKLOADS = {
    "tiny_256": dict(M=256, N=256, K=256, g=256, seed=0, outlier_count=4,
                     outlier_factor=20.0, w_std=0.02),
    "dit_attn_4096x3072x3072": dict(M=4096, N=3072, K=3072, g=256, seed=1,
                                    outlier_frac=0.01, outlier_factor=30.0, w_std=0.02,
                                    bias_std=0.01),
    "dit_mlp_4608x3840x10240": dict(M=4608, N=10240, K=3840, g=256, seed=2,
                                    dist="student_t", w_std=0.015),
    "peft_lora_8192x12288x3072_r64": dict(M=8192, N=12288, K=3072, g=256, seed=3,
                                          outlier_frac=0.01, outlier_factor=30.0,
                                          w_std=0.02, lora_rank=64, lora_std=0.01,
                                          lora_scale=1.0),
    "quarot_16384x4096x4096": dict(M=16384, N=4096, K=4096, g=256, seed=4,
                                   outlier_frac=0.02, outlier_factor=50.0, w_std=0.02,
                                   bias_std=0.01),
}


def make_grad_case(M, N, K, g=256, seed=0, dy_std=0.01, outlier_frac=0.0, outlier_count=None,
                   outlier_factor=1.0, w_std=0.02, ld_pad=0, name="grad") -> Case:
    """Output gradient dy [M, N] (in ``x``; ``ld_pad`` extra columns make it a strided view's
    parent) and the frozen layer's weight W [N, K]."""
    gen = torch.Generator("cpu").manual_seed(seed)
    dy = _normal(gen, (M, N + ld_pad), dy_std)
    count = outlier_count if outlier_count is not None else int(round(outlier_frac * N))
    cols = torch.randperm(N, generator=gen)[:count]
    if count:
        dy[:, cols] *= outlier_factor
    W = _normal(gen, (N, K), w_std).to(torch.bfloat16)
    return Case(name, M, N, K, g, dy.to(torch.bfloat16), W,
                extra={"outlier_cols": cols, "seed": seed, "grad": True, "ld_pad": ld_pad})


# Input-gradient workloads: the attention projection and the PEFT feed-forward layer run
# backwards (dy has the layer's N output features, dx its K input features).
GRAD_WORKLOADS = {
    "grad_dit_attn_4096x3072x3072": dict(M=4096, N=3072, K=3072, g=256, seed=5,
                                         outlier_frac=0.01, outlier_factor=30.0),
    "grad_peft_8192x12288x3072": dict(M=8192, N=12288, K=3072, g=256, seed=6,
                                      outlier_frac=0.01, outlier_factor=30.0),
}


def make_attn_case(B, L, H, D=128, g=256, seed=0, k_offset=3.0, name="attn") -> Case:
    """Self-attention inputs q, k, v [B, L, H, D] bf16 (q in ``x``, k in ``W``, v in
    extra["v"]); the keys carry a per-channel offset (the bias smooth_k removes)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _normal(gen, (B, L, H, D))
    k = _normal(gen, (B, L, H, D)) + k_offset * _normal(gen, (1, 1, H, D))
    v = _normal(gen, (B, L, H, D))
    return Case(name, L, H, D, g, q.to(torch.bfloat16), k.to(torch.bfloat16),
                extra={"v": v.to(torch.bfloat16), "attn": True, "B": B, "seed": seed})


# Attention workloads: the DiT joint attention of the linear workloads' model (Flux.1: 24
# heads of 128 over 4608 joint tokens).
ATTN_WORKLOADS = {
    "attn_flux_b1_l4608_h24_d128": dict(B=1, L=4608, H=24, D=128, g=256, seed=7),
}


def workload(name: str, g: int | None = None, M: int | None = None) -> Case:
    """Build one of the named workloads. ``g`` overrides the Hadamard group (the QuaRot
    sweep runs 64, 128, 256); ``M`` overrides the token count (smaller samples)."""
    if name in ATTN_WORKLOADS:
        kw = dict(ATTN_WORKLOADS[name])
        if g is not None:
            kw["g"] = g
        if M is not None:
            kw["L"] = M
        return make_attn_case(name=name, **kw)
    if name.startswith("fp8_"):
        # the FP8 (e4m3) variant runs on the same inputs as the int8 workload it names
        case = workload(name[len("fp8_"):], g=g, M=M)
        case.name = name
        case.extra["fp8"] = True
        return case
    grad = name in GRAD_WORKLOADS
    kw = dict(GRAD_WORKLOADS[name] if grad else WORKLOADS[name])
    if g is not None:
        kw["g"] = g
    if M is not None:
        kw["M"] = M
    if grad:
        return make_grad_case(name=name, **kw)
    case = make_case(name=name, **kw)
    if name.startswith("dit_mlp"):
        # the down projection: W_down [K_up, N_up] drawn after the up projection's tensors
        gen = torch.Generator("cpu").manual_seed(kw["seed"] + 1000)
        case.extra["W_down"] = _normal(gen, (kw["K"], kw["N"]), kw["w_std"]).to(torch.bfloat16)
    return case
