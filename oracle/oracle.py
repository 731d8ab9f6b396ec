"""CPU oracle for the Wan-style video-VAE decoder residual-block hot path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports this module and shares no code with it.

The arithmetic primitives live in ``oracle.c`` (fp64, compiled into
``liboracle.so`` by :func:`build`); this module marshals numpy float64 arrays
in the logical NCDHW order (batch 1, stored as [C, T, H, W]) and composes the
primitives into the residual block and the decoder trunk exactly as the block
is defined:

* norm + SiLU (TensorRT-LLM issue #19309, "Feature, motivation and proposed
  scope": decoder residual norm1/norm2 and norm_out are channel normalisation,
  affine scaling and SiLU);
* causal 3x3x3 conv with zero front frames and a one-pixel zero border
  (FastVideo Wan2.2 VAE decoder README, "Limits": bf16 operands, fp32
  accumulation; temporal caching named in the TensorRT-LLM issue's scope);
* residual block h = x + conv2(A2(conv1(A1(x)))), with a 1x1x1 shortcut conv
  on the raw input when the channel count changes;
* nearest 2x upsample followed by a per-frame 3x3 conv between stages, and
  (optionally) a temporal 2x upsample after the first two of them, giving
  4T - 3 video frames;
* the trunk: conv_in, three (2 res blocks, upsample conv) stages, 2 res blocks,
  norm_out + SiLU + causal conv to 12 channels and a 2x2 pixel shuffle into
  the 3-channel video (FastVideo README intro: 48 latent channels, 16x16
  spatial compression).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

EPS = 1e-12


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            D = ctypes.POINTER(ctypes.c_double)
            i = ctypes.c_int
            lib.orc_silu.restype = ctypes.c_double
            lib.orc_silu.argtypes = [ctypes.c_double]
            lib.orc_norm_silu.argtypes = [D, D, D, D, i, ctypes.c_long, ctypes.c_double, i]
            lib.orc_causal_conv3d.argtypes = [D, D, D, D, D] + [i] * 9
            lib.orc_causal_conv3d_at.argtypes = [D, D, D, D, D] + [i] * 11
            lib.orc_upsample_nearest2x.argtypes = [D, D, i, i, i, i]
            lib.orc_pixel_shuffle2x2.argtypes = [D, D, i, i, i, i]
            _lib = lib
    return _lib


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def nthreads() -> int:
    return max(1, os.cpu_count() or 1)


# ----------------------------------------------------------------- primitives
def silu(s: float) -> float:
    return _L().orc_silu(float(s))


def norm_silu(x, gamma, beta, eps: float = EPS, apply_silu: bool = True):
    """x: [C, T, H, W] (or [C, nvox]) -> same shape.  See oracle.c."""
    x = _f64(x)
    C = x.shape[0]
    y = np.empty_like(x)
    g, b = _f64(gamma), _f64(beta)
    assert g.shape == (C,) and b.shape == (C,)
    _L().orc_norm_silu(_p(x), _p(y), _p(g), _p(b), C, x.size // C, eps, int(apply_silu))
    return y


def causal_conv3d(x, wt, bias=None, cache=None, threads: int | None = None):
    """x: [Cin, T, H, W]; wt: [Cout, Cin, KT, KH, KW]; cache: [Cin, KT-1, H, W] or None."""
    x, wt, bias, cache = _f64(x), _f64(wt), _f64(bias), _f64(cache)
    Cin, T, H, W = x.shape
    Cout, Cin2, KT, KH, KW = wt.shape
    assert Cin2 == Cin and KH % 2 == 1 and KW % 2 == 1
    if cache is not None:
        assert cache.shape == (Cin, KT - 1, H, W)
    y = np.empty((Cout, T, H, W), dtype=np.float64)
    _L().orc_causal_conv3d(_p(x), _p(wt), _p(bias), _p(cache), _p(y), Cin, Cout, T, H, W,
                           KT, KH, KW, threads or nthreads())
    return y


def causal_conv3d_at(x, wt, bias, t: int, h: int, w: int, cache=None):
    """All Cout outputs of the causal conv at one voxel (t, h, w)."""
    x, wt, bias, cache = _f64(x), _f64(wt), _f64(bias), _f64(cache)
    Cin, T, H, W = x.shape
    Cout, _, KT, KH, KW = wt.shape
    yv = np.empty((Cout,), dtype=np.float64)
    _L().orc_causal_conv3d_at(_p(x), _p(wt), _p(bias), _p(cache), _p(yv), Cin, Cout, T, H, W,
                              KT, KH, KW, t, h, w)
    return yv


def upsample_nearest2x(x):
    x = _f64(x)
    C, T, H, W = x.shape
    y = np.empty((C, T, 2 * H, 2 * W), dtype=np.float64)
    _L().orc_upsample_nearest2x(_p(x), _p(y), C, T, H, W)
    return y


def pixel_shuffle2x2(x):
    x = _f64(x)
    C4, T, H, W = x.shape
    assert C4 % 4 == 0
    y = np.empty((C4 // 4, T, 2 * H, 2 * W), dtype=np.float64)
    _L().orc_pixel_shuffle2x2(_p(x), _p(y), C4 // 4, T, H, W)
    return y


# ---------------------------------------------------------------- composition
def resblock(x, p, threads: int | None = None):
    """Residual block.  p holds gamma1, beta1, w1, b1, gamma2, beta2, w2, b2 and,
    when Cin != Cout, ws, bs (the 1x1x1 shortcut)."""
    x = _f64(x)
    a1 = norm_silu(x, p["gamma1"], p["beta1"])
    h1 = causal_conv3d(a1, p["w1"], p["b1"], threads=threads)
    a2 = norm_silu(h1, p["gamma2"], p["beta2"])
    h2 = causal_conv3d(a2, p["w2"], p["b2"], threads=threads)
    if p.get("ws") is not None:
        skip = causal_conv3d(x, p["ws"], p["bs"], threads=threads)
    else:
        skip = x
    return h2 + skip


def temporal_upsample2x(x, first_chunk: bool = True):
    """Temporal 2x upsample of the causal decoder, shape only (nearest in time).

    The pages fix only the frame counts: latents [1, 48, T, ...] decode to
    4T - 3 video frames (FastVideo Wan2.2 VAE decoder README, opening section:
    4x temporal compression, video [1, 3, 4T - 3, 704, 1248]).  Read as two
    2x steps, each keeping the decode's first frame once (the causal first
    frame has no predecessor to pair with) and turning every later frame into
    two consecutive copies: T frames -> 2T - 1, and twice -> 4T - 3.  A chunk
    of a streaming decode that is not the first (first_chunk=False) holds no
    first frame, so all of its T frames double: T -> 2T.  x: [C, T, H, W]."""
    x = _f64(x)
    src = []
    for t in range(x.shape[1]):
        src += [t] if (t == 0 and first_chunk) else [t, t]
    return np.ascontiguousarray(x[:, src])


def upsample_conv(x, wt, bias, threads: int | None = None):
    """Nearest 2x upsample, then a per-frame 3x3 conv (KT = 1) with zero border."""
    return causal_conv3d(upsample_nearest2x(x), wt, bias, threads=threads)


def head(h, gamma, beta, wt, bias, threads: int | None = None):
    """norm_out + SiLU, causal conv to 12 channels, 2x2 pixel shuffle -> [3, T, 2H, 2W]."""
    a = norm_silu(h, gamma, beta)
    return pixel_shuffle2x2(causal_conv3d(a, wt, bias, threads=threads))


def trunk(z, params, threads: int | None = None, trace: dict | None = None,
          temporal: bool = False, first_chunk: bool = True):
    """Decoder trunk.  params: 'conv_in' -> (w, b); 'stages' -> list of dicts
    {'blocks': [resblock params...], 'up': (w, b) or None}; 'head' -> dict
    gamma, beta, w, b.  Returns the video [3, T', 2H', 2W'].  If ``trace`` is a
    dict, each layer's output is stored in it under its name.

    temporal=True adds the temporal 2x upsample (temporal_upsample2x) after the
    upsample convs of the first two stages, so the video has 4T - 3 frames
    (4T for a continuing chunk, first_chunk=False) instead of T.  Which two of
    the three upsamplings carry it is a reading: the pages give the frame
    count, not the place."""
    h = causal_conv3d(z, *params["conv_in"], threads=threads)
    if trace is not None:
        trace["conv_in"] = h
    for s, st in enumerate(params["stages"]):
        for r, bp in enumerate(st["blocks"]):
            h = resblock(h, bp, threads=threads)
            if trace is not None:
                trace[f"s{s}.b{r}"] = h
        if st["up"] is not None:
            h = upsample_conv(h, *st["up"], threads=threads)
            if temporal and s < 2:
                h = temporal_upsample2x(h, first_chunk)
            if trace is not None:
                trace[f"s{s}.up"] = h
    hp = params["head"]
    return head(h, hp["gamma"], hp["beta"], hp["w"], hp["b"], threads=threads)
