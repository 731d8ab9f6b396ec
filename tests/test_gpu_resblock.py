"""Residual block, upsample conv and decoder trunk vs the oracle (GPU)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, sample_voxels, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


def resblock_at(x, p, t, h, w):
    """Oracle block output at one voxel from the crop that determines it: frames
    t-4..t and a 2-pixel border (two stacked causal 3x3x3 convs).  Where the crop
    meets the tensor's edge the zero padding is the real one; elsewhere the
    crop's own padding only reaches outputs that are not read."""
    _, T, H, W = x.shape
    t0, h0, h1, w0, w1 = max(0, t - 4), max(0, h - 2), min(H, h + 3), max(0, w - 2), min(W, w + 3)
    y = O.resblock(x[:, t0:t + 1, h0:h1, w0:w1], p, threads=8)
    return y[:, t - t0, h - h0, w - w0]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_resblock_tiny(dtype):
    """Tiny res block: x [64, 2, 16, 16], two (norm + SiLU + conv 64->64) stages + identity."""
    x, p = synth.tiny_resblock(bf16=dtype == torch.bfloat16)
    blk = B.PackedResBlock(p, dtype)
    y = B.resblock(to_cl(x, dtype), blk)
    assert_close(from_cl(y), O.resblock(x, p), dtype, "tiny res block")


@pytest.mark.parametrize("cin,cout", [(256, 256), (256, 128), (128, 64), (64, 128), (512, 512)])
def test_resblock_reduced(cin, cout):
    """512 -> 512 runs its convs on clusters of two CTAs that split the channels and
    swap the RMS partial sums over distributed shared memory."""
    x, p = synth.resblock_input(cin=cin, cout=cout, T=3, H=11, W=19, seed=cin + cout)
    blk = B.PackedResBlock(p)
    y = B.resblock(to_cl(x), blk)
    assert_close(from_cl(y), O.resblock(x, p), torch.bfloat16, f"{cin}->{cout}")


@pytest.mark.parametrize("cout", [256, 128])
def test_resblock_full_size_sampled(cout):
    """Res block 256 -> 256 (and the 256 -> 128 shortcut variant) at [256, 4, 176, 312]."""
    x, p = synth.resblock_input(cin=256, cout=cout, T=4, H=176, W=312, seed=0)
    blk = B.PackedResBlock(p)
    y = B.resblock(to_cl(x), blk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    # 256 voxels: corners and edges, the seams of the 16 x 16 CTA tiles (rows
    # 15 | 16, columns 15 | 16), the two 8-row MMA sub-tiles of a tile (rows
    # 7 | 8), the last frame, and uniformly drawn voxels
    seams = {(t, h, w) for t in (0, 3) for h in (7, 8, 15, 16, 167, 168, 175)
             for w in (15, 16, 303, 304, 311)}
    pts = sorted(set(sample_voxels(4, 176, 312, 256 - len(seams), seed=3)) | seams)
    got = np.stack([yc[t, h, w].double().numpy() for (t, h, w) in pts], 1)
    ref = np.stack([resblock_at(x, p, t, h, w) for (t, h, w) in pts], 1)
    assert_close(got, ref, torch.bfloat16, f"res block 256->{cout}")
    assert torch.isfinite(yc).all()
    assert B.device_error() == 0


@pytest.mark.parametrize("cin,cout,H,W", [(128, 64, 6, 10), (64, 128, 5, 9), (512, 256, 4, 8),
                                          (256, 128, 9, 21)])
def test_upsample_conv(cin, cout, H, W):
    """Nearest 2x + 3x3 conv via the four phase kernels vs the oracle's dense definition."""
    g = torch.Generator().manual_seed(cin)
    x = synth.normal(g, (cin, 2, H, W))
    w, b = synth.conv_params(g, cout, cin, 1, 3, 3)
    pk = B.prepack_upsample_conv(w.cuda().bfloat16(), b.cuda())
    y = B.upsample_conv(to_cl(x), pk)
    assert y.shape == (2, 2 * H, 2 * W, cout)
    assert_close(from_cl(y), O.upsample_conv(x, w, b), torch.bfloat16, "upsample conv")


def test_upsample_conv_f32():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(64, 2, 5, 7, generator=g)
    w = torch.randn(32, 64, 1, 3, 3, generator=g) / 24.0
    b = 0.1 * torch.randn(32, generator=g)
    pk = B.prepack_upsample_conv(w.cuda(), b.cuda(), torch.float32)
    y = B.upsample_conv(to_cl(x, torch.float32), pk)
    assert_close(from_cl(y), O.upsample_conv(x, w, b), torch.float32, "upsample conv fp32")


def test_upsample_conv_full_size_sampled():
    """The trunk's 512 -> 256 upsample conv at [512, 4, 88, 156] -> [256, 4, 176, 312], sampled."""
    g = torch.Generator().manual_seed(21)
    x = synth.normal(g, (512, 4, 88, 156))
    w, b = synth.conv_params(g, 256, 512, 1, 3, 3)
    pk = B.prepack_upsample_conv(w.cuda().bfloat16(), b.cuda())
    y = B.upsample_conv(to_cl(x), pk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    pts = sample_voxels(4, 176, 312, 24, seed=4)
    got = np.stack([yc[t, h, ww].double().numpy() for (t, h, ww) in pts], 1)
    ref = []
    for (t, h, ww) in pts:
        # the output pixel depends on a 2x2 low-res window: crop, upsample, conv, read the centre
        h0, w0 = max(0, h // 2 - 1), max(0, ww // 2 - 1)
        h1, w1 = min(88, h // 2 + 2), min(156, ww // 2 + 2)
        crop = x[:, t:t + 1, h0:h1, w0:w1]
        yy = O.upsample_conv(crop, w, b)
        hb, wb = h - 2 * h0, ww - 2 * w0
        edge_ok = (h0 == 0 or hb >= 1) and (h1 == 88 or hb <= 2 * (h1 - h0) - 2) and \
                  (w0 == 0 or wb >= 1) and (w1 == 156 or wb <= 2 * (w1 - w0) - 2)
        assert edge_ok
        ref.append(yy[:, 0, hb, wb])
    assert_close(got, np.stack(ref, 1), torch.bfloat16, "upsample conv full size")
    assert B.device_error() == 0


def _trunk_case(T, H, W, widths, zc=48, seed=0):
    z, params = synth.trunk_input(T=T, H=H, W=W, widths=widths, zc=zc, seed=seed)
    tr = B.PackedTrunk(params)
    video = B.decode_trunk(z[None].cuda().bfloat16().contiguous(), tr)
    return z, params, video


def test_trunk_reduced_width_end_to_end():
    z, params, video = _trunk_case(T=3, H=3, W=5, widths=(128, 128, 64, 64))
    assert video.shape == (1, 3, 3, 48, 80)
    ref = O.trunk(z, params)
    assert_close(video[0].float().cpu().double().numpy(), ref, torch.bfloat16, "trunk reduced")


@pytest.mark.slow
def test_trunk_full_width_end_to_end():
    z, params, video = _trunk_case(T=2, H=4, W=6, widths=synth.TRUNK_WIDTHS)
    ref = O.trunk(z, params)
    assert_close(video[0].float().cpu().double().numpy(), ref, torch.bfloat16, "trunk full width")


def test_trunk_full_size_properties():
    """The trunk at full size (latents [1, 48, 4, 44, 78]): finite, deterministic, and
    causal bit for bit."""
    z, params = synth.trunk_input(T=4, H=44, W=78, seed=0)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    v0 = B.decode_trunk(zd, tr)
    v1 = B.decode_trunk(zd, tr)
    assert v0.shape == (1, 3, 4, 704, 1248)
    assert torch.isfinite(v0.float()).all()
    assert torch.equal(v0, v1)
    z2 = zd.clone()
    z2[:, :, 3] = torch.randn(1, 48, 44, 78, generator=torch.Generator().manual_seed(9)).bfloat16().cuda()
    v2 = B.decode_trunk(z2, tr)
    assert torch.equal(v0[:, :, :3], v2[:, :, :3])
    assert not torch.equal(v0[:, :, 3], v2[:, :, 3])
    assert B.device_error() == 0


@pytest.mark.parametrize("chunks", [(2, 4), (3, 3), (2, 2, 2)])
def test_trunk_chunked_decode_equals_whole(chunks):
    """Decoding the latents chunk by chunk, each causal conv reading its two
    front frames from the previous chunk's cache, gives the whole decode's
    video bit for bit (reduced widths, T = 6)."""
    T = sum(chunks)
    z, params = synth.trunk_input(T=T, H=3, W=5, widths=(128, 128, 64, 64), seed=3)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    whole = B.decode_trunk(zd, tr)
    stream = B.TrunkStream(tr, 3, 5)
    parts, t0 = [], 0
    for n in chunks:
        parts.append(stream.decode(zd[:, :, t0:t0 + n].contiguous()))
        t0 += n
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=2), whole)
    assert B.device_error() == 0


def test_trunk_chunked_decode_full_size():
    """Full widths and frames (latents [1, 48, 8, 44, 78]) in two chunks of 4
    against one decode of all 8 frames, bit for bit; the first chunk's video
    also equals a fresh 4-frame decode."""
    z, params = synth.trunk_input(T=8, H=44, W=78, seed=1)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    whole = B.decode_trunk(zd, tr)
    stream = B.TrunkStream(tr, 44, 78)
    a = stream.decode(zd[:, :, :4].contiguous())
    b = stream.decode(zd[:, :, 4:].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a, whole[:, :, :4])
    assert torch.equal(b, whole[:, :, 4:])
    assert torch.equal(a, B.decode_trunk(zd[:, :, :4].contiguous(), tr))
    assert B.device_error() == 0


def test_trunk_cuda_graph_replay():
    """The trunk captured once as a CUDA graph replays to the direct decode's
    video, also after new latents are copied into its input buffer."""
    z, params = synth.trunk_input(T=3, H=3, W=5, widths=(128, 128, 64, 64), seed=4)
    z2, _ = synth.trunk_input(T=3, H=3, W=5, widths=(128, 128, 64, 64), seed=5)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    zd2 = z2[None].cuda().bfloat16().contiguous()
    g = B.TrunkGraph(tr, zd.clone())
    assert torch.equal(g.replay().clone(), B.decode_trunk(zd, tr))
    g.z.copy_(zd2)
    assert torch.equal(g.replay().clone(), B.decode_trunk(zd2, tr))
    assert B.device_error() == 0


def test_resblock_128_many_waves_sampled():
    """Res block 128 -> 128 on [128, 4, 256, 320] (1,280 tiles per conv, conv1
    with the fused norm2).  256 sampled voxels against the oracle."""
    x, p = synth.resblock_input(cin=128, cout=128, T=4, H=256, W=320, seed=5)
    blk = B.PackedResBlock(p)
    y = B.resblock(to_cl(x), blk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    seams = {(t, h, c) for t in (0, 3) for h in (0, 7, 8, 31, 32) for c in (0, 15, 16, 319)}
    pts = sorted(set(sample_voxels(4, 256, 320, 256 - len(seams), seed=9)) | seams)
    got = np.stack([yc[t, h, c].double().numpy() for (t, h, c) in pts], 1)
    ref = np.stack([resblock_at(x, p, t, h, c) for (t, h, c) in pts], 1)
    assert_close(got, ref, torch.bfloat16, "res block 128 many waves")
    assert B.device_error() == 0


def test_trunk_timed_decode_equals_plain_and_records_every_launch():
    """wvae_decode_trunk_timed (the benchmark's per-launch timing) enqueues the
    same work as wvae_decode_trunk: the same video bit for bit, and an event
    pair around each of the 22 launches (the event clock ticks every ~2 us, so
    a small launch may read 0; the total is positive)."""
    z, params = synth.trunk_input(T=2, H=3, W=5, widths=(128, 128, 64, 64), seed=6)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    plain = B.decode_trunk(zd, tr)
    n = B.trunk_launches()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
    timed = B.decode_trunk(zd, tr, events=ev)
    torch.cuda.synchronize()
    assert torch.equal(plain, timed)
    durations = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n)]
    assert n == 22 and all(d >= 0 for d in durations) and sum(durations) > 0
    assert B.device_error() == 0
