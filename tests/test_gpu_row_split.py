"""The row split on the device (GPU): one decode divided by latent rows into
slabs that each carry one halo row per side, run through the library's
row-slab steps, with the halo rows filled between launches.  On one GPU the
ranks are emulated in one process: their slabs step in lockstep and the halo
rows are copied between them where the multi-GPU path exchanges them with
NCCL (video_diffusion_vae_b200/shard.py: decode_rows).  No kernel waits on
another.  The assembled video is checked against the oracle and against the
whole decode."""
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import shard
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3])
def test_row_split_vs_oracle(world):
    z, params = synth.trunk_input(T=3, H=6, W=5, widths=(128, 128, 64, 64), seed=37)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    video = shard.decode_rows_emulated(zd, tr, world)
    torch.cuda.synchronize()
    assert video.shape == (1, 3, 3, 96, 80)
    assert_close(video[0].float().cpu().double().numpy(), O.trunk(z, params), torch.bfloat16,
                 f"row split x{world}")
    whole = B.decode_trunk(zd, tr)
    assert torch.equal(video, whole), (video.float() - whole.float()).abs().max().item()
    assert B.device_error() == 0


@pytest.mark.parametrize("world", [2, 4])
def test_row_split_full_size_equals_whole(world):
    """Latents [1, 48, 4, 44, 78], full widths, split over 2 and 4 slabs (22 / 11
    latent rows each): the assembled video equals the whole decode's."""
    z, params = synth.trunk_input(T=4, H=44, W=78, seed=0)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    video = shard.decode_rows_emulated(zd, tr, world)
    whole = B.decode_trunk(zd, tr)
    torch.cuda.synchronize()
    assert video.shape == whole.shape == (1, 3, 4, 704, 1248)
    assert torch.equal(video, whole), (video.float() - whole.float()).abs().max().item()
    assert B.device_error() == 0


def test_row_split_one_row_slabs():
    """Three latent rows over three slabs: every slab holds one own row between
    two halo rows at stage 0 (and 8 at stage 3); the assembled video equals the
    whole decode and the oracle."""
    z, params = synth.trunk_input(T=2, H=3, W=4, widths=(128, 128, 64, 64), seed=43)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    video = shard.decode_rows_emulated(zd, tr, 3)
    whole = B.decode_trunk(zd, tr)
    torch.cuda.synchronize()
    assert torch.equal(video, whole)
    assert_close(video[0].float().cpu().double().numpy(), O.trunk(z, params), torch.bfloat16,
                 "one-row slabs")
    assert B.device_error() == 0
