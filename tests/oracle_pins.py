"""Pin checks for the CPU oracle, written so a planted mistake can be fed through them.

Each check takes an object exposing the oracle's functions (the real module, or
a copy with one function replaced by a mistaken variant) and raises
AssertionError when the oracle disagrees with something other than itself: a
hand-derived closed form (tests/golden/), a library routine on a special case,
brute force on a tiny input, or an invariant of the definition.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _floats(s):
    return [float(v) for v in s.split(",")]


def _kv(tok):
    k, v = tok.split("=", 1)
    return k, v


def load_norm_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "norm_silu_closed_form.txt")):
        if line.startswith("case "):
            d = dict(_kv(t) for t in line.split()[2:])
            cases.append(d)
    return cases


# ------------------------------------------------------------------- norm-SiLU
def check_norm_golden(O):
    for d in load_norm_cases():
        C = int(d["C"])
        x = np.array(_floats(d["x"])).reshape(C, 1)
        y = O.norm_silu(x, np.array(_floats(d["gamma"])), np.array(_floats(d["beta"])),
                        apply_silu=bool(int(d["silu"])))
        np.testing.assert_allclose(y.reshape(-1), _floats(d["y"]), rtol=1e-14, atol=1e-15)


def check_norm_unit_rms(O):
    rng = np.random.default_rng(1)
    C = 48
    x = rng.standard_normal((C, 2, 3, 5)) * rng.uniform(0.5, 2, (C, 1, 1, 1))
    y = O.norm_silu(x, np.ones(C), np.zeros(C), apply_silu=False)
    np.testing.assert_allclose((y ** 2).sum(0), C, rtol=1e-12)


def check_norm_scale_invariance(O):
    rng = np.random.default_rng(2)
    C = 16
    x = rng.standard_normal((C, 1, 4, 4))
    g, b = 1 + rng.standard_normal(C) * 0.3, rng.standard_normal(C) * 0.3
    np.testing.assert_allclose(O.norm_silu(7.5 * x, g, b), O.norm_silu(x, g, b), rtol=1e-12, atol=1e-14)


def check_norm_library(O):
    """F.normalize (eps clamps the norm) * sqrt(C) * gamma + beta, then F.silu."""
    rng = np.random.default_rng(3)
    C = 64
    x = rng.standard_normal((C, 2, 3, 4))
    x[:, 0, 0, 0] = 0.0              # eps clamp: all-zero voxel
    x[:, 0, 0, 1] = 1e-300            # sum of squares underflows to 0 -> clamp
    g, b = 1 + rng.standard_normal(C) * 0.3, rng.standard_normal(C) * 0.3
    xt = torch.from_numpy(x)
    ref = F.normalize(xt, dim=0, eps=1e-12) * math.sqrt(C) * torch.from_numpy(g).view(C, 1, 1, 1) \
        + torch.from_numpy(b).view(C, 1, 1, 1)
    ref = F.silu(ref).numpy()
    np.testing.assert_allclose(O.norm_silu(x, g, b), ref, rtol=1e-12, atol=1e-14)


def check_silu_limits(O):
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    assert abs(O.silu(-40.0)) < 1e-15
    np.testing.assert_allclose(O.silu(math.log(3.0)), 0.75 * math.log(3.0), rtol=1e-15)


# ---------------------------------------------------------------- causal conv
def load_conv_golden():
    rows = {}
    for line in open(os.path.join(GOLDEN, "causal_conv3d_hand.txt")):
        if line.startswith(("ones", "delta")):
            name, t, vals = line.split()
            rows.setdefault(name, {})[int(t.split("=")[1])] = _floats(vals)
    return rows


def check_conv_golden(O):
    g = load_conv_golden()
    x = np.ones((1, 2, 3, 3))
    w = np.ones((1, 1, 3, 3, 3))
    y = O.causal_conv3d(x, w, np.zeros(1))
    for t in (0, 1):
        np.testing.assert_array_equal(y[0, t].reshape(-1), g["ones"][t])
    x = np.zeros((1, 2, 2, 2))
    x[0, 0, 0, 0] = 1.0
    w = np.zeros((1, 1, 3, 3, 3))
    for kt in range(3):
        for kh in range(3):
            for kw in range(3):
                w[0, 0, kt, kh, kw] = 100 * kt + 10 * kh + kw
    y = O.causal_conv3d(x, w, np.zeros(1))
    for t in (0, 1):
        np.testing.assert_array_equal(y[0, t].reshape(-1), g["delta"][t])


def torch_causal_conv(x, w, b, cache=None):
    """Library routine: zero-pad (front frames, border) then F.conv3d, in float64."""
    KT, KH, KW = w.shape[2:]
    xt = torch.from_numpy(np.ascontiguousarray(x))[None]
    if cache is not None:
        xt = torch.cat([torch.from_numpy(cache)[None], xt], dim=2)
        pt = 0
    else:
        pt = KT - 1
    xt = F.pad(xt, ((KW - 1) // 2, (KW - 1) // 2, (KH - 1) // 2, (KH - 1) // 2, pt, 0))
    return F.conv3d(xt, torch.from_numpy(w), None if b is None else torch.from_numpy(b))[0].numpy()


def check_conv_library(O):
    rng = np.random.default_rng(4)
    for (Cin, Cout, T, H, W, k) in [(5, 7, 3, 6, 9, (3, 3, 3)), (4, 3, 2, 5, 4, (1, 3, 3)),
                                    (6, 2, 3, 4, 5, (1, 1, 1)), (3, 4, 4, 3, 3, (3, 1, 1))]:
        x = rng.standard_normal((Cin, T, H, W))
        w = rng.standard_normal((Cout, Cin) + k)
        b = rng.standard_normal(Cout)
        np.testing.assert_allclose(O.causal_conv3d(x, w, b), torch_causal_conv(x, w, b),
                                   rtol=1e-12, atol=1e-12)
    # with the previous chunk's cached frames in place of the zero frames
    x = rng.standard_normal((3, 2, 4, 5))
    cache = rng.standard_normal((3, 2, 4, 5))
    w = rng.standard_normal((2, 3, 3, 3, 3))
    b = rng.standard_normal(2)
    np.testing.assert_allclose(O.causal_conv3d(x, w, b, cache=cache),
                               torch_causal_conv(x, w, b, cache=cache), rtol=1e-12, atol=1e-12)


def brute_conv(x, w, b):
    """Seven nested loops straight from the definition (tiny inputs only)."""
    Cin, T, H, W = x.shape
    Cout, _, KT, KH, KW = w.shape
    y = np.zeros((Cout, T, H, W))
    for o in range(Cout):
        for t in range(T):
            for h in range(H):
                for ww in range(W):
                    acc = b[o]
                    for i in range(Cin):
                        for kt in range(KT):
                            for kh in range(KH):
                                for kw in range(KW):
                                    ts, hs, ws = t + kt - (KT - 1), h + kh - (KH - 1) // 2, ww + kw - (KW - 1) // 2
                                    if 0 <= ts < T and 0 <= hs < H and 0 <= ws < W:
                                        acc += w[o, i, kt, kh, kw] * x[i, ts, hs, ws]
                    y[o, t, h, ww] = acc
    return y


def check_conv_brute(O):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 3, 3, 2))
    w = rng.standard_normal((3, 2, 3, 3, 3))
    b = rng.standard_normal(3)
    np.testing.assert_allclose(O.causal_conv3d(x, w, b), brute_conv(x, w, b), rtol=1e-12, atol=1e-12)
    # single-voxel form against the full form
    y = O.causal_conv3d(x, w, b)
    for (t, h, ww) in [(0, 0, 0), (2, 1, 1), (1, 2, 0)]:
        np.testing.assert_allclose(O.causal_conv3d_at(x, w, b, t, h, ww), y[:, t, h, ww], rtol=1e-13)


def check_conv_invariants(O):
    rng = np.random.default_rng(6)
    Cin, Cout, T, H, W = 3, 4, 4, 5, 6
    x = rng.standard_normal((Cin, T, H, W))
    w = rng.standard_normal((Cout, Cin, 3, 3, 3))
    b = rng.standard_normal(Cout)
    y = O.causal_conv3d(x, w, b)
    # causality: changing frame t leaves outputs before t unchanged, bit for bit
    for t in range(1, T):
        x2 = x.copy()
        x2[:, t] += rng.standard_normal((Cin, H, W))
        y2 = O.causal_conv3d(x2, w, b)
        assert np.array_equal(y2[:, :t], y[:, :t])
        assert not np.allclose(y2[:, t], y[:, t])
    # zero weights give the bias exactly
    y0 = O.causal_conv3d(x, np.zeros_like(w), b)
    assert np.array_equal(y0, np.broadcast_to(b.reshape(-1, 1, 1, 1), y0.shape))
    # linearity in the weights
    w2 = rng.standard_normal(w.shape)
    lhs = O.causal_conv3d(x, 2.0 * w - 3.0 * w2, None)
    rhs = 2.0 * O.causal_conv3d(x, w, None) - 3.0 * O.causal_conv3d(x, w2, None)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-11)
    # translation equivariance away from the border (shift by one column)
    xs = np.zeros_like(x)
    xs[..., 1:] = x[..., :-1]
    ys = O.causal_conv3d(xs, w, b)
    np.testing.assert_allclose(ys[..., 2:-1], y[..., 1:-2], rtol=1e-12, atol=1e-12)


# ------------------------------------------------- upsample, pixel shuffle
def check_upsample(O):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 2, 4, 5))
    y = O.upsample_nearest2x(x)
    ref = F.interpolate(torch.from_numpy(x), scale_factor=2, mode="nearest").numpy()
    assert np.array_equal(y, ref)
    for i in (0, 1):
        for j in (0, 1):
            assert np.array_equal(y[:, :, i::2, j::2], x)


def check_pixel_shuffle(O):
    rows = {}
    for line in open(os.path.join(GOLDEN, "pixel_shuffle_hand.txt")):
        if line.startswith("y "):
            _, c, vals = line.split()
            rows[int(c.split("=")[1])] = _floats(vals)
    x = np.arange(1, 9, dtype=np.float64).reshape(8, 1, 1, 1)
    y = O.pixel_shuffle2x2(x)
    for c, vals in rows.items():
        np.testing.assert_array_equal(y[c, 0].reshape(-1), vals)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((12, 2, 3, 4))
    ref = F.pixel_shuffle(torch.from_numpy(x).permute(1, 0, 2, 3), 2).permute(1, 0, 2, 3).numpy()
    assert np.array_equal(O.pixel_shuffle2x2(x), ref)
    assert np.isclose(O.pixel_shuffle2x2(x).sum(), x.sum())


# ------------------------------------------------------------ composition
def torch_resblock(x, p):
    """The residual block built from library routines (float64, CPU)."""
    def A(v, g, b):
        v = F.normalize(v, dim=0, eps=1e-12) * math.sqrt(v.shape[0]) * g.view(-1, 1, 1, 1) + b.view(-1, 1, 1, 1)
        return F.silu(v)

    def conv(v, w, b):
        return torch.from_numpy(torch_causal_conv(v.numpy(), w.numpy(), b.numpy()))
    x = torch.as_tensor(x, dtype=torch.float64)
    q = {k: torch.as_tensor(v, dtype=torch.float64) for k, v in p.items()}
    h = conv(A(x, q["gamma1"], q["beta1"]), q["w1"], q["b1"])
    h = conv(A(h, q["gamma2"], q["beta2"]), q["w2"], q["b2"])
    skip = conv(x, q["ws"], q["bs"]) if "ws" in q else x
    return (h + skip).numpy()


def check_resblock_library(O, synth):
    x, p = synth.resblock_input(cin=16, cout=16, T=3, H=5, W=7, seed=3)
    np.testing.assert_allclose(O.resblock(x, p), torch_resblock(x, p), rtol=1e-10, atol=1e-10)
    x, p = synth.resblock_input(cin=16, cout=8, T=2, H=4, W=6, seed=4)
    np.testing.assert_allclose(O.resblock(x, p), torch_resblock(x, p), rtol=1e-10, atol=1e-10)


def check_resblock_identity(O):
    """Zero conv weights and biases: the block returns x exactly."""
    rng = np.random.default_rng(9)
    C = 8
    x = rng.standard_normal((C, 2, 3, 4))
    z = np.zeros((C, C, 3, 3, 3))
    p = dict(gamma1=np.ones(C), beta1=np.zeros(C), w1=z, b1=np.zeros(C),
             gamma2=np.ones(C), beta2=np.zeros(C), w2=z, b2=np.zeros(C))
    assert np.array_equal(O.resblock(x, p), x)


# ------------------------------------------------------ temporal upsample
def load_temporal_golden():
    src, frames = [], []
    for line in open(os.path.join(GOLDEN, "temporal_upsample_hand.txt")):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] in ("first", "next"):
            src.append((f[0] == "first", int(f[1]), [int(v) for v in f[2:]]))
        elif f[0] == "frames":
            frames.append((int(f[1]), int(f[2])))
    return src, frames


def check_temporal_golden(O):
    """Hand-listed source frames: frame index t carried in the data itself."""
    src, _ = load_temporal_golden()
    for first, T, want in src:
        x = np.arange(T, dtype=np.float64).reshape(1, T, 1, 1) * np.ones((2, T, 2, 3))
        y = O.temporal_upsample2x(x, first_chunk=first)
        assert y.shape == (2, len(want), 2, 3)
        assert np.array_equal(y[0, :, 0, 0], np.array(want, dtype=np.float64))
        assert np.array_equal(y, y[:1].repeat(2, 0))    # every channel and pixel alike


def check_temporal_library(O):
    """torch.repeat_interleave on the time axis, less the first copy of frame 0
    for a decode's first chunk; streaming: chunk by chunk equals all at once."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((3, 5, 2, 4))
    rep = torch.repeat_interleave(torch.from_numpy(x), 2, dim=1).numpy()
    assert np.array_equal(O.temporal_upsample2x(x, first_chunk=True), rep[:, 1:])
    assert np.array_equal(O.temporal_upsample2x(x, first_chunk=False), rep)
    parts = [O.temporal_upsample2x(x[:, :2], True), O.temporal_upsample2x(x[:, 2:], False)]
    assert np.array_equal(np.concatenate(parts, 1), O.temporal_upsample2x(x, True))


def check_temporal_trunk_frames(O, synth):
    """The trunk with temporal upsampling: 4T - 3 frames (the pages' count,
    tests/golden/temporal_upsample_hand.txt), the first frame equal to the
    trunk without it at T = 1, and causal in upsampled time: changing latent
    frame t >= 1 leaves video frames before 4t - 3 unchanged and changes frame
    4t - 3."""
    _, frames = load_temporal_golden()
    for T, n in frames:
        if T <= 4:
            z, params = synth.trunk_input(T=T, H=2, W=2, widths=(8, 8, 8, 8), zc=4, seed=T)
            assert O.trunk(z, params, temporal=True).shape[1] == n
    z, params = synth.trunk_input(T=1, H=2, W=3, widths=(8, 8, 8, 8), zc=4, seed=6)
    assert np.array_equal(O.trunk(z, params, temporal=True), O.trunk(z, params))
    z, params = synth.trunk_input(T=3, H=2, W=2, widths=(8, 8, 8, 8), zc=4, seed=7)
    v0 = O.trunk(z, params, temporal=True)
    for t in (1, 2):
        z2 = z.clone()
        z2[:, t] += 1.0
        v1 = O.trunk(z2, params, temporal=True)
        assert np.array_equal(v0[:, :4 * t - 3], v1[:, :4 * t - 3])
        assert not np.allclose(v0[:, 4 * t - 3], v1[:, 4 * t - 3])


def torch_trunk_temporal(z, params):
    """The trunk with temporal upsampling from library routines (float64, CPU):
    repeat_interleave in time after the first two upsample convs."""
    def conv(v, w, b):
        return torch.from_numpy(torch_causal_conv(v.numpy(), w.double().numpy(), b.double().numpy()))
    h = conv(z.double(), *params["conv_in"])
    for s, st in enumerate(params["stages"]):
        for bp in st["blocks"]:
            h = torch.from_numpy(torch_resblock(h, bp))
        if st["up"] is not None:
            h = conv(F.interpolate(h, scale_factor=2, mode="nearest"), *st["up"])
            if s < 2:
                h = torch.repeat_interleave(h, 2, dim=1)[:, 1:]
    hp = params["head"]
    C = h.shape[0]
    a = F.silu(F.normalize(h, dim=0, eps=1e-12) * math.sqrt(C) * hp["gamma"].double().view(-1, 1, 1, 1)
               + hp["beta"].double().view(-1, 1, 1, 1))
    o = conv(a, hp["w"], hp["b"])
    return F.pixel_shuffle(o.permute(1, 0, 2, 3), 2).permute(1, 0, 2, 3).numpy()


def check_trunk_temporal_library(O, synth):
    z, params = synth.trunk_input(T=3, H=2, W=3, widths=(16, 16, 8, 8), zc=6, seed=8)
    np.testing.assert_allclose(O.trunk(z, params, temporal=True), torch_trunk_temporal(z, params),
                               rtol=1e-9, atol=1e-9)


ALL_CHECKS = [check_norm_golden, check_norm_unit_rms, check_norm_scale_invariance,
              check_norm_library, check_silu_limits, check_conv_golden, check_conv_library,
              check_conv_brute, check_conv_invariants, check_upsample, check_pixel_shuffle,
              check_resblock_identity, check_temporal_golden, check_temporal_library]


def torch_trunk(z, params):
    """The decoder trunk built from library routines (float64, CPU)."""
    def conv(v, w, b):
        return torch.from_numpy(torch_causal_conv(v.numpy(), w.double().numpy(), b.double().numpy()))
    h = conv(z.double(), *params["conv_in"])
    for st in params["stages"]:
        for bp in st["blocks"]:
            h = torch.from_numpy(torch_resblock(h, bp))
        if st["up"] is not None:
            h = conv(F.interpolate(h, scale_factor=2, mode="nearest"), *st["up"])
    hp = params["head"]
    C = h.shape[0]
    a = F.silu(F.normalize(h, dim=0, eps=1e-12) * math.sqrt(C) * hp["gamma"].double().view(-1, 1, 1, 1)
               + hp["beta"].double().view(-1, 1, 1, 1))
    o = conv(a, hp["w"], hp["b"])
    return F.pixel_shuffle(o.permute(1, 0, 2, 3), 2).permute(1, 0, 2, 3).numpy()


def check_trunk_library(O, synth):
    z, params = synth.trunk_input(T=2, H=3, W=4, widths=(16, 16, 8, 8), zc=6, seed=5)
    np.testing.assert_allclose(O.trunk(z, params), torch_trunk(z, params), rtol=1e-9, atol=1e-9)
