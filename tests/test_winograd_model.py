"""Tolerance study of a Winograd F(2x2, 3x3) conv against the direct conv (CPU).

The page-3 decoder computes its convs as products of Winograd-transformed
weights and activations (FastVideo "Wan2.2 VAE decoder" README, "Performance
and memory"); the library's kernels compute the direct definition.  Before a
Winograd kernel is built, these tests fix (1) that the model in
tests/winograd_model.py is the same conv as the oracle's direct one in exact
arithmetic, and (2) what rounding the transformed operands to the tensor
cores' 16-bit types costs, with the activations rounded to bf16 at the same
tensor boundaries as the library's bf16 path, against the fp64 oracle:

    workload                          direct        Winograd, bf16 V/U   Winograd, fp16 V/U
    res block 256 ch [2,12,14]        1.9e-3 / 1.5e-2   2.8e-3 / 1.8e-2   1.9e-3 / 1.4e-2
    trunk, latents [1,48,2,2,3]       4.3e-3 / 2.1e-2   8.0e-3 / 3.6e-2   4.4e-3 / 2.2e-2
    (rel-L2 / max|err| over std; the bars are 1e-2 / 5e-2)

bf16 transformed operands stay inside the bars but take 80 % of the rel-L2
budget over the trunk; fp16 operands (the same tensor-core rate) are as
accurate as the direct conv.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import winograd_model as WM
from video_diffusion_vae_b200 import synth

REL_BAR, MAX_BAR = 1e-2, 5e-2


def bf(a):
    return WM.round_to(a, torch.bfloat16)


def f64(t):
    return np.asarray(t.double().numpy() if isinstance(t, torch.Tensor) else t, dtype=np.float64)


def errors(got, ref):
    return (float(np.linalg.norm(got - ref) / np.linalg.norm(ref)),
            float(np.abs(got - ref).max() / ref.std()))


def conv_for(operand):
    if operand == "direct":
        return lambda a, w, b: O.causal_conv3d(a, f64(w), f64(b))
    return lambda a, w, b: WM.causal_conv3d_winograd(a, f64(w), f64(b), operand=operand)


def resblock_bf16(x, p, conv):
    """The res block with the bf16 path's rounding points: both conv inputs
    (the norm-SiLU activations) are bf16; the residual stream is not rounded."""
    a1 = bf(O.norm_silu(x, p["gamma1"], p["beta1"]))
    h1 = conv(a1, p["w1"], p["b1"])
    a2 = bf(O.norm_silu(h1, p["gamma2"], p["beta2"]))
    skip = O.causal_conv3d(x, f64(p["ws"]), f64(p["bs"])) if p.get("ws") is not None else x
    return conv(a2, p["w2"], p["b2"]) + skip


def trunk_bf16(z, params, conv):
    """The trunk with the bf16 path's rounding points: every conv input is bf16,
    the fp32 residual stream is not rounded, the video is bf16.  Only the
    3x3x3 convs change with `conv`; the upsample convs stay direct."""
    h = conv(f64(z), *params["conv_in"])
    for st in params["stages"]:
        for bp in st["blocks"]:
            h = resblock_bf16(h, bp, conv)
        if st["up"] is not None:
            h = O.upsample_conv(bf(h), f64(st["up"][0]), f64(st["up"][1]))
    hp = params["head"]
    a = bf(O.norm_silu(h, hp["gamma"], hp["beta"]))
    return bf(O.pixel_shuffle2x2(conv(a, hp["w"], hp["b"])))


@pytest.mark.parametrize("shape", [(3, 4, 3, 5, 7, 3), (2, 3, 2, 6, 6, 1), (4, 2, 1, 1, 1, 3),
                                   (5, 3, 2, 3, 2, 3), (6, 5, 4, 9, 4, 3)])
def test_winograd_form_equals_direct_conv(shape):
    """Exact arithmetic: the F(2x2, 3x3) form is the direct causal conv, ragged
    tiles included (odd H and W, a 1x1 frame, KT = 1)."""
    Cin, Cout, T, H, W, KT = shape
    rng = np.random.default_rng(sum(shape))
    x = rng.standard_normal((Cin, T, H, W))
    w = rng.standard_normal((Cout, Cin, KT, 3, 3))
    b = rng.standard_normal(Cout)
    ref = O.causal_conv3d(x, w, b)
    got = WM.causal_conv3d_winograd(x, w, b)
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


def test_winograd_transforms_of_a_delta():
    """A delta filter at tap (kh, kw) shifts the input: out[h, w] = x[h+kh-1, w+kw-1]."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 1, 5, 6))
    for kh in range(3):
        for kw in range(3):
            w = np.zeros((1, 1, 1, 3, 3))
            w[0, 0, 0, kh, kw] = 1.0
            y = WM.causal_conv3d_winograd(x, w)
            xp = np.pad(x[0, 0], 1)
            np.testing.assert_allclose(y[0, 0], xp[kh:kh + 5, kw:kw + 6], atol=1e-14)


def test_resblock_operand_precision():
    x, p = synth.resblock_input(cin=256, cout=256, T=2, H=12, W=14, seed=1)
    x = f64(x)
    ref = O.resblock(x, p)
    e = {op: errors(bf(resblock_bf16(x, p, conv_for(op))), ref)
         for op in ("direct", torch.bfloat16, torch.float16)}
    for rel, mx in e.values():
        assert rel <= REL_BAR and mx <= MAX_BAR
    assert e[torch.bfloat16][0] > 1.3 * e["direct"][0]      # bf16 transforms cost accuracy
    assert e[torch.float16][0] < 1.1 * e["direct"][0]       # fp16 transforms do not


def test_trunk_operand_precision():
    z, params = synth.trunk_input(T=2, H=2, W=3, seed=2)
    ref = O.trunk(z, params)
    e = {op: errors(trunk_bf16(z, params, conv_for(op)), ref)
         for op in ("direct", torch.bfloat16, torch.float16)}
    for rel, mx in e.values():
        assert rel <= REL_BAR and mx <= MAX_BAR
    assert e[torch.bfloat16][0] > 1.5 * e["direct"][0]
    assert e[torch.bfloat16][0] > 0.6 * REL_BAR             # most of the budget
    assert e[torch.float16][0] < 1.1 * e["direct"][0]
