"""The decoder trunk against the oracle where only large layers reach (GPU).

Three kinds of comparison, all at the bf16 path's tolerances
(rel-L2 <= 1e-2, max |err| <= 5e-2 x std of the reference):

* Every output element at sizes where the last stage runs more tiles than
  the 148 SMs, so persistent CTAs take a second tile: latents [1, 48, 3, 12, 20]
  put stage 3 at 96 x 160 x 3 frames = 180 tiles of 16 x 16 voxels (and the
  stage-2 -> 3 upsample conv at 48 x 80 x 3 frames x 4 phases = 180 tiles).
  With 256 channels at stage 3 one accumulator fills TMEM, so the conv2 of
  block 0 and the upsample conv (fused norm + fp32 raw output) release it
  after epilogue pass 1; with 128 channels two accumulators alternate and the
  epilogue of one tile overlaps the next tile's main loop.
* Sampled pixels of the full-size trunk (latents [1, 48, 4, 44, 78], the
  benchmark's workload and launch configuration) against oracle values stored
  by tests/golden/make_trunk_full_size_samples.py; the max-error bound uses
  the std of the whole oracle video, stored beside the samples.
* The streaming decode (chunks of latent frames carrying the causal caches)
  against the oracle's decode of all frames at once.
"""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import REL_L2_BF16, MAX_ABS_BF16, assert_close
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "trunk_full_size_samples.txt")


def _decode(z, params):
    tr = B.PackedTrunk(params)
    video = B.decode_trunk(z[None].cuda().bfloat16().contiguous(), tr)
    torch.cuda.synchronize()
    return tr, video


@pytest.mark.parametrize("widths", [(64, 64, 64, 256), (64, 64, 64, 128)])
def test_trunk_multi_tile_vs_oracle(widths):
    z, params = synth.trunk_input(T=3, H=12, W=20, widths=widths, seed=31)
    _, video = _decode(z, params)
    assert video.shape == (1, 3, 3, 192, 320)
    ref = O.trunk(z, params)
    assert_close(video[0].float().cpu().double().numpy(), ref, torch.bfloat16,
                 f"trunk widths {widths}")
    assert B.device_error() == 0


def _read_golden(path=GOLDEN):
    meta, rows = {}, []
    with open(path) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) == 2:
                meta[parts[0]] = float(parts[1])
            else:
                rows.append((int(parts[0]), int(parts[1]), int(parts[2]), int(parts[3]),
                             float(parts[4])))
    assert len(rows) == int(meta["count"])
    return meta, rows


def test_trunk_full_size_vs_oracle_samples():
    """The benchmark's decode (latents [1, 48, 4, 44, 78], seed 0, widths
    512/512/256/128) at ~8,500 pixels: every (channel, frame) at the crossings
    of 18 rows and 16 columns on tile seams and frame edges, plus 5,000 drawn
    uniformly.  Covers what only full-size layers run: several tiles per CTA at
    every stage, the 512-channel layers' CTA pairs with the early accumulator
    release, and the wave-balanced tile shapes."""
    meta, rows = _read_golden()
    z, params = synth.trunk_input(T=4, H=44, W=78, seed=0)
    _, video = _decode(z, params)
    assert video.shape == (1, 3, 4, 704, 1248)
    v = video[0].float().cpu()
    idx = torch.tensor([r[:4] for r in rows])
    got = v[idx[:, 0], idx[:, 1], idx[:, 2], idx[:, 3]].double().numpy()
    ref = np.array([r[4] for r in rows])
    assert np.isfinite(got).all()
    d = got - ref
    rel = np.linalg.norm(d) / np.linalg.norm(ref)
    mx = np.abs(d).max() / meta["std"]
    assert rel <= REL_L2_BF16, f"rel L2 {rel:.3e}"
    assert mx <= MAX_ABS_BF16, f"max |err| / std {mx:.3e}"
    # the whole video's scale matches the oracle's (a wholesale error elsewhere
    # in the frame would show here)
    assert abs(v.double().std().item() / meta["std"] - 1.0) < 1e-2
    assert B.device_error() == 0


@pytest.mark.parametrize("T,H,W,widths,chunks", [
    (6, 3, 5, (128, 128, 64, 64), (2, 4)),
    (6, 3, 5, (128, 128, 64, 64), (2, 2, 2)),
    (6, 12, 20, (64, 64, 64, 128), (3, 3)),   # 180 stage-3 tiles per chunk
])
def test_trunk_chunked_decode_vs_oracle(T, H, W, widths, chunks):
    """Chunk by chunk on the GPU (each causal conv reading its front frames
    from the previous chunk's cache) against the oracle's whole decode."""
    z, params = synth.trunk_input(T=T, H=H, W=W, widths=widths, seed=17)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    stream = B.TrunkStream(tr, H, W)
    parts, t0 = [], 0
    for n in chunks:
        parts.append(stream.decode(zd[:, :, t0:t0 + n].contiguous()))
        t0 += n
    torch.cuda.synchronize()
    got = torch.cat(parts, dim=2)[0].float().cpu().double().numpy()
    assert_close(got, O.trunk(z, params), torch.bfloat16, f"chunked {chunks}")
    assert B.device_error() == 0


# ------------------------------------------- video decode with 4T - 3 frames
@pytest.mark.parametrize("T,H,W,widths", [
    (3, 3, 5, (128, 128, 64, 64)),
    (2, 6, 10, (64, 64, 64, 128)),   # stage 3: 5 frames x 60 tiles of 16 x 16 at 96 x 160
])
def test_video_decode_vs_oracle(T, H, W, widths):
    """The temporal 2x steps ride in the first two upsample convs' epilogues:
    video [1, 3, 4T - 3, 16H, 16W] against the oracle's decode with them."""
    z, params = synth.trunk_input(T=T, H=H, W=W, widths=widths, seed=23)
    tr = B.PackedTrunk(params)
    v = B.decode_video(z[None].cuda().bfloat16().contiguous(), tr)
    torch.cuda.synchronize()
    assert v.shape == (1, 3, 4 * T - 3, 16 * H, 16 * W)
    ref = O.trunk(z, params, temporal=True)
    assert_close(v[0].float().cpu().double().numpy(), ref, torch.bfloat16, f"video T={T}")
    assert B.device_error() == 0


@pytest.mark.parametrize("chunks", [(2, 3), (2, 2, 2)])
def test_video_stream_vs_oracle(chunks):
    """Chunk by chunk: the first chunk keeps its first frame once (4T - 3
    frames), later chunks double every frame (4T); together the oracle's
    whole decode."""
    T = sum(chunks)
    z, params = synth.trunk_input(T=T, H=3, W=5, widths=(128, 128, 64, 64), seed=29)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    stream = B.VideoStream(tr, 3, 5)
    parts, t0 = [], 0
    for i, n in enumerate(chunks):
        parts.append(stream.decode(zd[:, :, t0:t0 + n].contiguous()))
        assert parts[-1].shape[2] == (4 * n - 3 if i == 0 else 4 * n)
        t0 += n
    torch.cuda.synchronize()
    got = torch.cat(parts, dim=2)[0].float().cpu().double().numpy()
    assert_close(got, O.trunk(z, params, temporal=True), torch.bfloat16, f"video chunks {chunks}")
    assert B.device_error() == 0


def test_video_decode_full_size_properties():
    """Latents [1, 48, 4, 44, 78] -> video [1, 3, 13, 704, 1248]: finite; two
    chunks of 2 equal the whole decode bit for bit; the first video frame
    (which sees only latent frame 0 at every stage) is the plain trunk's first
    frame; changing latent frame 3 leaves video frames 0..8 (before 4*3 - 3)
    unchanged."""
    z, params = synth.trunk_input(T=4, H=44, W=78, seed=0)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    v = B.decode_video(zd, tr)
    assert v.shape == (1, 3, 13, 704, 1248)
    assert torch.isfinite(v.float()).all()
    stream = B.VideoStream(tr, 44, 78)
    a = stream.decode(zd[:, :, :2].contiguous())
    b = stream.decode(zd[:, :, 2:].contiguous())
    assert torch.equal(torch.cat([a, b], 2), v)
    plain = B.decode_trunk(zd, tr)
    rel = ((v[:, :, 0].float() - plain[:, :, 0].float()).norm() / plain[:, :, 0].float().norm()).item()
    assert rel < 1e-3, rel
    z2 = zd.clone()
    z2[:, :, 3] = 0
    v2 = B.decode_video(z2, tr)
    assert torch.equal(v[:, :, :9], v2[:, :, :9])
    assert not torch.equal(v[:, :, 9], v2[:, :, 9])
    assert B.device_error() == 0


# ------------------------------------------------------------- edge cases
def test_trunk_and_video_single_latent_frame():
    """T = 1: every causal conv sees only its current frame (two zero frames in
    front), and the video decode with temporal upsampling keeps the single
    frame once (4T - 3 = 1): both equal the oracle's trunk."""
    z, params = synth.trunk_input(T=1, H=3, W=5, widths=(128, 128, 64, 64), seed=41)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    v = B.decode_trunk(zd, tr)
    vv = B.decode_video(zd, tr)
    torch.cuda.synchronize()
    assert v.shape == vv.shape == (1, 3, 1, 48, 80)
    ref = O.trunk(z, params)
    assert_close(v[0].float().cpu().double().numpy(), ref, torch.bfloat16, "trunk T=1")
    assert_close(vv[0].float().cpu().double().numpy(), ref, torch.bfloat16, "video T=1")
    assert B.device_error() == 0


VIDEO_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                            "trunk_video_full_size_samples.txt")


def test_video_decode_full_size_vs_oracle_samples():
    """The 4T - 3 decode at full size: latents [1, 48, 4, 44, 78] (seed 0) ->
    video [1, 3, 13, 704, 1248], at ~10,000 pixels (every channel on frames
    0, 1, 2, 5, 9, 12 at the crossings of 18 rows and 16 columns on tile
    seams and frame edges, plus 5,000 uniform) against oracle values stored
    by tests/golden/make_trunk_full_size_samples.py --video; the max-error
    bound uses the std of the whole oracle video.  Covers the temporal 2x
    steps written by the upsample convs' epilogues at full size (stages 1-3
    on 7 and 13 frames, several tiles per CTA everywhere)."""
    meta, rows = _read_golden(VIDEO_GOLDEN)
    z, params = synth.trunk_input(T=4, H=44, W=78, seed=0)
    tr = B.PackedTrunk(params)
    video = B.decode_video(z[None].cuda().bfloat16().contiguous(), tr)
    torch.cuda.synchronize()
    assert video.shape == (1, 3, 13, 704, 1248)
    v = video[0].float().cpu()
    idx = torch.tensor([r[:4] for r in rows])
    got = v[idx[:, 0], idx[:, 1], idx[:, 2], idx[:, 3]].double().numpy()
    ref = np.array([r[4] for r in rows])
    assert np.isfinite(got).all()
    d = got - ref
    rel = np.linalg.norm(d) / np.linalg.norm(ref)
    mx = np.abs(d).max() / meta["std"]
    assert rel <= REL_L2_BF16, f"rel L2 {rel:.3e}"
    assert mx <= MAX_ABS_BF16, f"max |err| / std {mx:.3e}"
    assert abs(v.double().std().item() / meta["std"] - 1.0) < 1e-2
    assert B.device_error() == 0


def test_video_decode_193_frames_whole_equals_streamed():
    """The pages' video length in one call: latents [1, 48, 49, 44, 78] ->
    video [1, 3, 193, 704, 1248].  The whole decode's stage-3 tensors hold
    5.4 G elements (offsets past 2^31; ~50 GB of workspace); the streamed
    decode (chunks of 5 + 11 x 4 latent frames) never more than 0.6 G.  Each
    chunk's video equals its frames of the whole decode bit for bit."""
    z, params = synth.trunk_input(T=49, H=44, W=78, seed=5)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    whole = B.decode_video(zd, tr)
    assert whole.shape == (1, 3, 193, 704, 1248)
    stream = B.VideoStream(tr, 44, 78)
    t0 = 0
    for n in [5] + [4] * 11:
        part = stream.decode(zd[:, :, t0:t0 + n].contiguous())
        f0 = 0 if t0 == 0 else 4 * t0 - 3
        assert part.shape[2] == (4 * n - 3 if t0 == 0 else 4 * n)
        assert torch.equal(part, whole[:, :, f0:f0 + part.shape[2]]), f"chunk at latent frame {t0}"
        t0 += n
    assert t0 == 49
    assert torch.isfinite(whole).all()
    assert B.device_error() == 0
