"""The Winograd F(2x2, 3x3) form of the causal 3x3x3 conv against the oracle's
direct conv (GPU).  The CPU tolerance study (tests/test_winograd_model.py)
shows that fp16 transformed operands keep the direct conv's accuracy, so the
bars are the bf16 path's own: rel-L2 <= 1e-2 and max |err| <= 5e-2 x std."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, sample_voxels, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cin,cout,T,H,W", [
    (64, 64, 2, 9, 17),      # odd H and W: the last tile row / column is ragged
    (64, 128, 3, 8, 16),
    (128, 256, 3, 13, 22),
    (64, 512, 2, 10, 12),    # two N tiles of 256
])
def test_winograd_conv_vs_oracle(cin, cout, T, H, W):
    x, w, b = synth.conv_input(cin=cin, cout=cout, T=T, H=H, W=W, seed=cin + cout + H)
    pk = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d_winograd(to_cl(x), pk)
    torch.cuda.synchronize()
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, f"winograd {cin}->{cout}")
    assert B.device_error() == 0


def test_winograd_conv_residual_and_fp32_weights():
    x, w, b = synth.conv_input(cin=64, cout=64, T=3, H=7, W=11, seed=41, bf16=False)
    xb = x.bfloat16().float()
    res = torch.randn(64, 3, 7, 11, generator=torch.Generator().manual_seed(42)).bfloat16().float()
    pk = B.prepack_conv_winograd(w.cuda(), b.cuda())          # fp32 weights in
    y = B.causal_conv3d_winograd(to_cl(xb), pk, residual=to_cl(res))
    ref = O.causal_conv3d(xb, w, b) + res.double().numpy()
    assert_close(from_cl(y), ref, torch.bfloat16, "winograd residual")


def test_winograd_conv_causality_bitwise():
    """Changing frame t leaves every output frame before t bit-identical."""
    x, w, b = synth.conv_input(cin=64, cout=64, T=4, H=9, W=14, seed=43)
    pk = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
    y0 = B.causal_conv3d_winograd(to_cl(x), pk)
    x2 = x.clone()
    x2[:, 2] = torch.randn(64, 9, 14, generator=torch.Generator().manual_seed(44)).bfloat16().float()
    y1 = B.causal_conv3d_winograd(to_cl(x2), pk)
    assert torch.equal(y0[:2], y1[:2])
    assert not torch.equal(y0[2], y1[2])


def test_winograd_conv_full_size_sampled():
    """512 -> 512 on [512, 4, 88, 156] (the config-2 conv), 256 sampled voxels
    (corners, edges, tile seams) against the oracle, and the whole output
    against the direct tensor-core conv at the same bars."""
    x, w, b = synth.conv_input(cin=512, cout=512, T=4, H=88, W=156, seed=0)
    wd, bd = w.cuda().bfloat16(), b.cuda()
    xd = to_cl(x)
    y = B.causal_conv3d_winograd(xd, B.prepack_conv_winograd(wd, bd))
    direct = B.causal_conv3d(xd, B.prepack_conv(wd, bd))
    torch.cuda.synchronize()
    yc = y.float().cpu()
    seams = {(t, h, c) for t in (0, 3) for h in (0, 1, 2, 15, 16, 87) for c in (0, 1, 2, 63, 64, 155)}
    pts = sorted(set(sample_voxels(4, 88, 156, 256 - len(seams), seed=6)) | seams)
    got = np.stack([yc[t, h, c].double().numpy() for (t, h, c) in pts], 1)
    ref = np.stack([O.causal_conv3d_at(x, w, b, t, h, c) for (t, h, c) in pts], 1)
    assert_close(got, ref, torch.bfloat16, "winograd 512 full size sampled")
    assert_close(y.float().cpu().double().numpy(), direct.float().cpu().double().numpy(),
                 torch.bfloat16, "winograd vs direct")
    assert B.device_error() == 0
