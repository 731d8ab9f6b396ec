"""Winograd F(2x2, 3x3) form of the causal 3x3x3 conv: a numerical model for
the tolerance study of the fast-algorithm conv (the page-3 decoder multiplies
Winograd-transformed weights and activations: FastVideo "Wan2.2 VAE decoder"
README, "Use" and "Performance and memory").

The algorithm is the minimal-filtering form of Lavin and Gray, "Fast
Algorithms for Convolutional Neural Networks" (CVPR 2016), section 4: for a
4x4 input tile d and a 3x3 filter g, the 2x2 output tile is
    Y = A^T [ (G g G^T) * (B^T d B) ] A        (* elementwise)
with the 4x4 tiles taken at stride 2.  The causal 3x3x3 conv applies it per
temporal tap kt and sums the sixteen elementwise products over the input
channels and the taps before the output transform, so a tensor-core kernel
runs sixteen GEMMs of K = KT * Cin.  Zero padding: two frames in front, one
pixel around the frame (the tiles of the last row / column read zeros past
the frame and their extra outputs are dropped).

`operand` models the precision of the transformed operands a kernel feeds to
the tensor cores: the transforms of bf16 activations and weights need more
bits than bf16 holds, so rounding them back to bf16 (or fp16) adds error that
the direct conv does not have.  Products are summed in float64 here; the
output is rounded by the caller.  This is test infrastructure: no kernel of
the library uses it.
"""
from __future__ import annotations

import numpy as np
import torch

# Lavin and Gray, F(2x2, 3x3): input transform B^T, filter transform G, output transform A^T.
BT = np.array([[1, 0, -1, 0],
               [0, 1, 1, 0],
               [0, -1, 1, 0],
               [0, 1, 0, -1]], dtype=np.float64)
G = np.array([[1, 0, 0],
              [0.5, 0.5, 0.5],
              [0.5, -0.5, 0.5],
              [0, 0, 1]], dtype=np.float64)
AT = np.array([[1, 1, 1, 0],
               [0, 1, -1, -1]], dtype=np.float64)


def round_to(a, dtype):
    """Round float64 values to a torch dtype (round to nearest even) and back."""
    if dtype is None:
        return a
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to(torch.float64).numpy()


def causal_conv3d_winograd(x, w, b=None, operand=None):
    """x [Cin, T, H, W], w [Cout, Cin, KT, 3, 3], b [Cout] or None -> [Cout, T, H, W].

    operand: None (exact), torch.bfloat16 or torch.float16: the precision of the
    transformed activations V and weights U."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Cin, T, H, W = x.shape
    Cout, _, KT, KH, KW = w.shape
    assert (KH, KW) == (3, 3)
    nh, nw = -(-H // 2), -(-W // 2)
    xp = np.zeros((Cin, T + KT - 1, 2 * nh + 2, 2 * nw + 2))
    xp[:, KT - 1:, 1:H + 1, 1:W + 1] = x
    d = np.lib.stride_tricks.sliding_window_view(xp, (4, 4), axis=(2, 3))[:, :, ::2, ::2]
    V = round_to(np.einsum("ab,ctijbd,ed->ctijae", BT, d, BT), operand)   # B^T d B
    U = round_to(np.einsum("ab,ockbd,ed->ockae", G, w, G), operand)       # G g G^T
    M = np.zeros((Cout, T, nh, nw, 4, 4))
    for kt in range(KT):
        M += np.einsum("ocae,ctijae->otijae", U[:, :, kt], V[:, kt:kt + T])
    Y = np.einsum("pa,otijae,qe->otipjq", AT, M, AT)                       # A^T M A
    y = Y.reshape(Cout, T, 2 * nh, 2 * nw)[:, :, :H, :W].copy()
    if b is not None:
        y += np.asarray(b, dtype=np.float64).reshape(-1, 1, 1, 1)
    return y
