"""Precision of the trunk's residual stream, studied on the CPU.

The bf16 path rounds every conv input (the norm-SiLU activations, the
upsample conv's input) to bf16 and keeps the residual stream - the raw
outputs of conv_in, of every res block and of every upsample conv - in fp32.
This model puts the same rounding points into the oracle's fp64 arithmetic
and compares the video with the exact one, for the fp32 stream and for a bf16
stream (the residual stream rounded to bf16 wherever it is stored):

    latents [1,48,2,2,3], full widths   fp32 stream 4.3e-3 / 2.1e-2   bf16 stream 6.2e-3 / 2.6e-2
    latents [1,48,4,4,6] (trunk_model)  fp32 stream 4.3e-3 / 2.1e-2   bf16 stream 6.5e-3 / 3.3e-2
    (rel-L2 / max|err| over std; the bars are 1e-2 / 5e-2)

The maximum error grows with the number of outputs, so at the full size a
bf16 stream would leave a thin margin under the max-error bar: the trunk keeps
the stream in fp32.
"""
import numpy as np
import torch

from oracle import oracle as O
from video_diffusion_vae_b200 import synth

REL_BAR, MAX_BAR = 1e-2, 5e-2


def bf(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float64).numpy()


def f64(t):
    return np.asarray(t.double().numpy() if isinstance(t, torch.Tensor) else t, dtype=np.float64)


def trunk_model(z, params, stream_bf16):
    """The trunk with the bf16 path's rounding points; stream_bf16 also rounds
    the stored residual stream."""
    keep = bf if stream_bf16 else (lambda a: a)
    h = keep(O.causal_conv3d(f64(z), *params["conv_in"]))
    for st in params["stages"]:
        for p in st["blocks"]:
            a1 = bf(O.norm_silu(h, p["gamma1"], p["beta1"]))
            h1 = O.causal_conv3d(a1, p["w1"], p["b1"])
            a2 = bf(O.norm_silu(h1, p["gamma2"], p["beta2"]))
            h = keep(O.causal_conv3d(a2, p["w2"], p["b2"]) + h)
        if st["up"] is not None:
            h = keep(O.upsample_conv(bf(h), *st["up"]))
    hp = params["head"]
    a = bf(O.norm_silu(h, hp["gamma"], hp["beta"]))
    return bf(O.pixel_shuffle2x2(O.causal_conv3d(a, hp["w"], hp["b"])))


def errors(got, ref):
    return (float(np.linalg.norm(got - ref) / np.linalg.norm(ref)),
            float(np.abs(got - ref).max() / ref.std()))


def test_residual_stream_precision():
    z, params = synth.trunk_input(T=2, H=2, W=3, seed=2)
    ref = O.trunk(z, params)
    f32 = errors(trunk_model(z, params, False), ref)
    b16 = errors(trunk_model(z, params, True), ref)
    assert f32[0] <= REL_BAR and f32[1] <= MAX_BAR
    assert b16[0] <= REL_BAR and b16[1] <= MAX_BAR
    assert b16[0] > 1.3 * f32[0] and b16[1] > f32[1]      # the bf16 stream costs accuracy
    assert f32[1] < 0.5 * MAX_BAR                         # the fp32 stream keeps half the bar free
