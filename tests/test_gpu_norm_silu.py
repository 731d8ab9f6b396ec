"""norm-SiLU kernel vs the oracle (GPU)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, sample_voxels, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("C", [8, 48, 64, 128, 256, 512, 1024])
def test_norm_silu_shapes(C, dtype):
    x, g, b = synth.norm_silu_input(C=C, T=2, H=5, W=7, seed=C)
    if dtype == torch.float32:
        x = x + 1e-3 * torch.randn(x.shape, generator=torch.Generator().manual_seed(1))
    y = B.norm_silu(to_cl(x, dtype), g.cuda(), b.cuda())
    assert_close(from_cl(y), O.norm_silu(x, g, b), dtype, f"C={C}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_norm_silu_clamp_edges(dtype):
    """All-zero and vanishing voxels take the eps clamp: output SiLU(beta)."""
    C = 64
    x, g, b = synth.norm_silu_input(C=C, T=1, H=3, W=4, seed=3)
    x = x.clone()
    x[:, 0, 0, 0] = 0.0
    x[:, 0, 1, 2] = 1e-30 if dtype == torch.float32 else 0.0
    x[:, 0, 2, 3] = 1e-20
    y = from_cl(B.norm_silu(to_cl(x, dtype), g.cuda(), b.cuda()))
    ref = O.norm_silu(x.to(dtype).double(), g, b)
    assert_close(y, ref, dtype, "clamp")
    np.testing.assert_allclose(y[:, 0, 0, 0], ref[:, 0, 0, 0], rtol=1e-2, atol=1e-2)


def test_norm_silu_in_place():
    x, g, b = synth.norm_silu_input(C=256, T=2, H=3, W=9, seed=5)
    xd = to_cl(x)
    ref = O.norm_silu(x, g, b)
    B.norm_silu(xd, g.cuda(), b.cuda(), out=xd)
    assert_close(from_cl(xd), ref, torch.bfloat16, "in place")


@pytest.mark.parametrize("shape", [(512, 4, 88, 156), (256, 4, 176, 312)])
def test_norm_silu_full_size_sampled(shape):
    C, T, H, W = shape
    x, g, b = synth.norm_silu_input(C=C, T=T, H=H, W=W, seed=0)
    y = B.norm_silu(to_cl(x), g.cuda(), b.cuda())
    torch.cuda.synchronize()
    pts = sample_voxels(T, H, W, 2048, seed=1)
    idx = tuple(np.array(pts).T)
    xs = x.permute(1, 2, 3, 0)[idx].T.contiguous()            # [C, n]
    ys = y.float().cpu()[idx].T.double().numpy()
    assert_close(ys, O.norm_silu(xs, g, b), torch.bfloat16, f"full {shape}")
    assert B.device_error() == 0


@pytest.mark.parametrize("C,T,H,W", [(512, 4, 87, 91), (64, 4, 176, 330), (1024, 2, 83, 89)])
def test_norm_silu_many_chunks_ragged(C, T, H, W):
    """Over 3 x 148 chunks of 64 KB (the 3-stage ring wraps around in every CTA)
    and a ragged last chunk; every voxel compared."""
    x, g, b = synth.norm_silu_input(C=C, T=T, H=H, W=W, seed=C + 7)
    y = B.norm_silu(to_cl(x), g.cuda(), b.cuda())
    assert_close(from_cl(y), O.norm_silu(x, g, b), torch.bfloat16, f"C={C}")
    assert B.device_error() == 0
