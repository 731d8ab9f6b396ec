"""Convs on CTA pairs at the tile counts that exercise the pair logic (GPU).

A conv with one N tile of 128 or 256 output channels per CTA runs on CTA
pairs that share M = 256 MMAs: the two CTAs take neighbouring spatial tiles
of the same (N tile, upsample phase), and when the count of spatial tiles is
odd the last pair's second CTA computes a copy of the last tile and writes
nothing.  These cases check the outputs against the oracle element by
element at odd and even tile counts, a single tile, several N tiles and the
upsample phases; writes outside the output are checked by the guard tests.
"""
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


def to_cl(x):
    return x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()


def from_cl(y):
    return y.float().cpu().permute(3, 0, 1, 2).double().numpy()


# spatial tiles per launch (16 x 16 tiles at 128 channels; 8 x 32 or 16 x 16 at 256):
# T=1, 16x16 -> 1 tile (the pair's second CTA only copies); T=3, 16x16 -> 3 (odd);
# T=2, 16x32 -> 4; T=1, 24x40 -> 2 x 3 = 6 at 16x16 (rows ragged), T=3, 24x40 -> 18
@pytest.mark.parametrize("cout", [128, 256])
@pytest.mark.parametrize("T,H,W", [(1, 16, 16), (3, 16, 16), (2, 16, 32), (3, 24, 40), (1, 9, 37)])
def test_pair_conv_tile_counts(cout, T, H, W):
    x, w, b = synth.conv_input(cin=64, cout=cout, T=T, H=H, W=W, seed=T * 100 + H + W + cout)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    torch.cuda.synchronize()
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, f"cout={cout} T={T} {H}x{W}")
    assert B.device_error() == 0


@pytest.mark.parametrize("T", [1, 3])
def test_pair_conv_two_n_tiles(T):
    """512 output channels without a fused norm: two 256-wide N tiles, each
    run by pairs (partners share the N tile)."""
    x, w, b = synth.conv_input(cin=128, cout=512, T=T, H=9, W=21, seed=5 + T)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    torch.cuda.synchronize()
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, f"cout=512 T={T}")
    assert B.device_error() == 0


@pytest.mark.parametrize("cin,cout,T,H,W", [(256, 128, 1, 5, 9), (256, 256, 3, 7, 11), (128, 256, 1, 16, 16)])
def test_pair_upsample_conv(cin, cout, T, H, W):
    """Upsample convs on pairs: partners share the phase (its 2 x 2 weights).
    These run the staged-store kernel (each warp's 32-channel chunks written
    with TMA stores of 16-voxel row segments; the ragged widths clip at W)."""
    g = torch.Generator().manual_seed(cin + cout + T)
    x = synth.normal(g, (cin, T, H, W))
    w, b = synth.conv_params(g, cout, cin, 1, 3, 3)
    pk = B.prepack_upsample_conv(w.cuda().bfloat16(), b.cuda())
    y = B.upsample_conv(to_cl(x), pk)
    torch.cuda.synchronize()
    assert y.shape == (T, 2 * H, 2 * W, cout)
    assert_close(from_cl(y), O.upsample_conv(x, w, b), torch.bfloat16, f"upsample {cin}->{cout} T={T}")
    assert B.device_error() == 0


@pytest.mark.parametrize("c,T,H,W", [(128, 1, 8, 16), (256, 3, 9, 17)])
def test_pair_resblock_odd_tiles(c, T, H, W):
    """A res block whose convs run on pairs with an odd tile count (fused
    norm, residual and raw outputs in the pair epilogues)."""
    x, p = synth.resblock_input(c, c, T, H, W, seed=c + T)
    blk = B.PackedResBlock(p)
    y = B.resblock(to_cl(x), blk)
    torch.cuda.synchronize()
    assert_close(from_cl(y), O.resblock(x, p), torch.bfloat16, f"resblock {c} T={T} {H}x{W}")
    assert B.device_error() == 0
