"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module only draws random numbers: it holds none of the decoder's
arithmetic.  Every tensor is drawn once on the CPU from a ``torch.Generator``
seeded per workload, in a fixed order (the input first, then each layer's
parameters in forward order: conv weight, conv bias; norm gamma, norm beta),
so both sides read the same bytes.

Distributions (``N(0, v)`` means variance ``v``):
  * activations / latents ~ N(0, 1) (the standalone norm workload multiplies
    channel c by a scale ~ U(0.5, 2));
  * conv weights ~ N(0, 1 / fan_in), fan_in = Cin * KT * KH * KW;
  * conv bias ~ N(0, 0.01); gamma ~ 1 + N(0, 0.1); beta ~ N(0, 0.1).
Values the GPU consumes in bf16 (activations, weights) are rounded to bf16
here, so the oracle sees exactly the numbers the kernels see.  gamma, beta and
bias stay fp32 (the kernels take them in fp32).

Logical shapes are batch-free NCDHW, i.e. [C, T, H, W]; conv weights are
PyTorch's [Cout, Cin, KT, KH, KW].
"""
from __future__ import annotations

import math

import torch

#: channel widths of the Wan2.2-shaped decoder trunk, one per stage
TRUNK_WIDTHS = (512, 512, 256, 128)
Z_CHANNELS = 48
VIDEO_CHANNELS = 3


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _round(t: torch.Tensor, bf16: bool) -> torch.Tensor:
    return t.to(torch.bfloat16).float() if bf16 else t


def normal(g, shape, var=1.0, bf16=True):
    return _round(torch.randn(*shape, generator=g) * math.sqrt(var), bf16)


def conv_params(g, cout, cin, kt, kh, kw, bf16=True):
    fan_in = cin * kt * kh * kw
    w = normal(g, (cout, cin, kt, kh, kw), 1.0 / fan_in, bf16)
    b = torch.randn(cout, generator=g) * math.sqrt(0.01)
    return w, b


def norm_params(g, c):
    gamma = 1.0 + torch.randn(c, generator=g) * math.sqrt(0.1)
    beta = torch.randn(c, generator=g) * math.sqrt(0.1)
    return gamma, beta


def resblock_params(g, cin, cout, bf16=True):
    p = {}
    p["gamma1"], p["beta1"] = norm_params(g, cin)
    p["w1"], p["b1"] = conv_params(g, cout, cin, 3, 3, 3, bf16)
    p["gamma2"], p["beta2"] = norm_params(g, cout)
    p["w2"], p["b2"] = conv_params(g, cout, cout, 3, 3, 3, bf16)
    if cin != cout:
        p["ws"], p["bs"] = conv_params(g, cout, cin, 1, 1, 1, bf16)
    return p


# ------------------------------------------------------------------ workloads
def tiny_resblock(bf16=True, seed=0, c=64, T=2, H=16, W=16):
    """Tiny res block: x [64, 2, 16, 16], two 64->64 stages, identity residual."""
    g = _gen(seed)
    x = normal(g, (c, T, H, W), 1.0, bf16)
    return x, resblock_params(g, c, c, bf16)


def norm_silu_input(C=512, T=4, H=88, W=156, seed=0):
    """Standalone norm-SiLU: x ~ N(0,1) * s_c with s_c ~ U(0.5, 2), bf16."""
    g = _gen(seed)
    x = torch.randn(C, T, H, W, generator=g)
    scale = 0.5 + 1.5 * torch.rand(C, generator=g)
    x = _round(x * scale.view(C, 1, 1, 1), True)
    gamma, beta = norm_params(g, C)
    return x, gamma, beta


def conv_input(cin=512, cout=512, T=4, H=88, W=156, seed=0, k=(3, 3, 3), bf16=True):
    """Causal conv3d workload: x ~ N(0,1), weights ~ N(0, 1/fan_in), bias ~ N(0, 0.01)."""
    g = _gen(seed)
    x = normal(g, (cin, T, H, W), 1.0, bf16)
    w, b = conv_params(g, cout, cin, *k, bf16=bf16)
    return x, w, b


def resblock_input(cin=256, cout=256, T=4, H=176, W=312, seed=0, bf16=True):
    """Full res block workload (cin == cout: identity residual; else 1x1x1 shortcut)."""
    g = _gen(seed)
    x = normal(g, (cin, T, H, W), 1.0, bf16)
    return x, resblock_params(g, cin, cout, bf16)


def trunk_input(T=4, H=44, W=78, widths=TRUNK_WIDTHS, zc=Z_CHANNELS, seed=0, blocks=2):
    """Wan2.2-shaped decoder trunk: z [48, T, H, W] and every layer's parameters.

    Layer order: conv_in; per stage: `blocks` res blocks, then (except the last
    stage) the upsample conv to the next width; then norm_out and the head conv
    to 12 channels (4 per video channel for the 2x2 pixel shuffle).
    """
    g = _gen(seed)
    z = normal(g, (zc, T, H, W), 1.0, True)
    params = {"conv_in": conv_params(g, widths[0], zc, 3, 3, 3), "stages": []}
    for s, c in enumerate(widths):
        blocks_p = [resblock_params(g, c, c) for _ in range(blocks)]
        up = conv_params(g, widths[s + 1], c, 1, 3, 3) if s + 1 < len(widths) else None
        params["stages"].append({"blocks": blocks_p, "up": up})
    gamma, beta = norm_params(g, widths[-1])
    w, b = conv_params(g, 4 * VIDEO_CHANNELS, widths[-1], 3, 3, 3)
    params["head"] = {"gamma": gamma, "beta": beta, "w": w, "b": b}
    return z, params
