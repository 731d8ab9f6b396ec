"""Causal conv3d (tcgen05 implicit GEMM and the fp32 path) vs the oracle (GPU)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, sample_voxels, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu


def _run(x, w, b, dtype, **kw):
    pk = B.prepack_conv(w.cuda().to(dtype), b.cuda(), dtype)
    return pk, B.causal_conv3d(to_cl(x, dtype), pk, **kw)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_tiny(dtype):
    """The tiny workload's conv: 64 -> 64, x [64, 2, 16, 16]."""
    x, w, b = synth.conv_input(cin=64, cout=64, T=2, H=16, W=16, seed=0, bf16=dtype == torch.bfloat16)
    _, y = _run(x, w, b, dtype)
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), dtype, "tiny")


@pytest.mark.parametrize("cout", [16, 64, 128, 256, 512])
def test_conv_ragged_tiles(cout):
    """H, W not multiples of the 8 x 16 tile; T = 3; several output widths."""
    x, w, b = synth.conv_input(cin=64, cout=cout, T=3, H=13, W=21, seed=cout)
    _, y = _run(x, w, b, torch.bfloat16)
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, f"cout={cout}")


@pytest.mark.parametrize("k", [(1, 3, 3), (1, 1, 1), (3, 3, 3)])
def test_conv_kernel_sizes_two_chunks(k):
    x, w, b = synth.conv_input(cin=128, cout=64, T=2, H=9, W=17, seed=7, k=k)
    _, y = _run(x, w, b, torch.bfloat16)
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, f"k={k}")


@pytest.mark.parametrize("dtype,cout", [(torch.bfloat16, 64), (torch.float32, 64), (torch.bfloat16, 128), (torch.bfloat16, 16)])
def test_conv_with_residual_norm_and_cache(dtype, cout):
    """cout 64 and 128: a group's window and its three row taps in one stage;
    cout 16: the column taps ride in N (the residual case runs the plain path)."""
    bf = dtype == torch.bfloat16
    x, w, b = synth.conv_input(cin=64, cout=cout, T=3, H=10, W=18, seed=11, bf16=bf)
    g = torch.Generator().manual_seed(12)
    res = torch.randn(cout, 3, 10, 18, generator=g)
    res = res.to(torch.bfloat16).float() if bf else res
    gamma = 1 + 0.3 * torch.randn(64, generator=g)
    beta = 0.3 * torch.randn(64, generator=g)
    cache = torch.randn(64, 2, 10, 18, generator=g)
    cache = cache.to(torch.bfloat16).float() if bf else cache
    pk = B.prepack_conv(w.cuda().to(dtype), b.cuda(), dtype)
    # residual
    y = B.causal_conv3d(to_cl(x, dtype), pk, residual=to_cl(res, dtype))
    assert_close(from_cl(y), O.causal_conv3d(x, w, b) + res.double().numpy(), dtype, "residual")
    # norm + SiLU before the conv (padding applies after the norm)
    y = B.causal_conv3d(to_cl(x, dtype), pk, norm=(gamma.cuda(), beta.cuda()))
    ref = O.causal_conv3d(O.norm_silu(x, gamma, beta), w, b)
    assert_close(from_cl(y), ref, dtype, "norm")
    # previous chunk's cached frames in place of the zero frames
    y = B.causal_conv3d(to_cl(x, dtype), pk, cache=to_cl(cache, dtype))
    assert_close(from_cl(y), O.causal_conv3d(x, w, b, cache=cache), dtype, "cache")


def test_conv_causality_bitwise():
    """Changing frame t leaves every output frame before t bit-identical."""
    x, w, b = synth.conv_input(cin=64, cout=128, T=4, H=9, W=20, seed=13)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y0 = B.causal_conv3d(to_cl(x), pk)
    x2 = x.clone()
    x2[:, 2] = torch.randn(64, 9, 20, generator=torch.Generator().manual_seed(14)).bfloat16().float()
    y1 = B.causal_conv3d(to_cl(x2), pk)
    assert torch.equal(y0[:2], y1[:2])
    assert not torch.equal(y0[2], y1[2])


def test_conv_full_size_sampled():
    """512 -> 512 on [512, 4, 88, 156] (full size); sampled voxels against the oracle."""
    x, w, b = synth.conv_input(cin=512, cout=512, T=4, H=88, W=156, seed=0)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    # 512 voxels: corners and edges, the seams of the 8 x 32 CTA tiles (rows
    # 7 | 8, columns 31 | 32), the two 4-row MMA sub-tiles of a tile (rows
    # 3 | 4), the ragged last tile column (128..155), every frame, and
    # uniformly drawn voxels
    seams = {(t, h, c) for t in range(4) for h in (3, 4, 7, 8, 83, 84, 87)
             for c in (31, 32, 127, 128, 155)}
    pts = sorted(set(sample_voxels(4, 88, 156, 512 - len(seams), seed=2)) | seams)
    got = np.stack([yc[t, h, ww].double().numpy() for (t, h, ww) in pts], 1)
    ref = np.stack([O.causal_conv3d_at(x, w, b, t, h, ww) for (t, h, ww) in pts], 1)
    assert_close(got, ref, torch.bfloat16, "512->512 full size sampled")
    assert torch.isfinite(yc).all()
    assert B.device_error() == 0


def test_conv_wide_tiles_sampled():
    """128 -> 128 on [128, 13, 40, 60]: with 148 SMs, CTA tiles of 8 x 32 voxels
    (130 tiles; each MMA sub-tile is 4 rows x 32 columns) need fewer waves than
    16 x 16 tiles (156), so this layer takes the wide shape, ragged in W."""
    T, H, W = 13, 40, 60
    x, w, b = synth.conv_input(cin=128, cout=128, T=T, H=H, W=W, seed=5)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    pts = set(sample_voxels(T, H, W, 40, seed=4))
    # both sub-tiles of a tile (rows 3 | 4), tile seams, the ragged last tile
    pts |= {(0, 3, 31), (0, 4, 0), (1, 7, 31), (2, 8, 32), (12, 35, 47), (12, 36, 48), (6, 20, 59)}
    pts = sorted(pts)
    got = np.stack([yc[t, h, ww].double().numpy() for (t, h, ww) in pts], 1)
    ref = np.stack([O.causal_conv3d_at(x, w, b, t, h, ww) for (t, h, ww) in pts], 1)
    assert_close(got, ref, torch.bfloat16, "wide tiles sampled")
    assert torch.isfinite(yc).all()
    assert B.device_error() == 0


def test_conv_epilogue_16_byte_aligned_buffers():
    """Output and residual 16- but not 32-byte aligned take the 128-bit
    epilogue accesses; the result is identical to the 256-bit path's."""
    T, H, W, cin, cout = 2, 9, 20, 64, 128
    x, w, b = synth.conv_input(cin=cin, cout=cout, T=T, H=H, W=W, seed=21)
    res = torch.randn(cout, T, H, W, generator=torch.Generator().manual_seed(22)).bfloat16().float()
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    xd, rd = to_cl(x), to_cl(res)
    y32 = B.causal_conv3d(xd, pk, residual=rd)
    n = T * H * W * cout
    obuf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    rbuf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    out16 = obuf[8:].view(T, H, W, cout)    # 16 bytes past a 256-byte boundary
    res16 = rbuf[8:].view(T, H, W, cout)
    res16.copy_(rd)
    assert out16.data_ptr() % 32 == 16 and res16.data_ptr() % 32 == 16
    B.causal_conv3d(xd, pk, residual=res16, out=out16)
    torch.cuda.synchronize()
    assert torch.equal(out16, y32)
    assert_close(from_cl(y32), O.causal_conv3d(x, w, b) + res.double().numpy(), torch.bfloat16, "res")


@pytest.mark.parametrize("cout", [128, 64])
def test_conv_many_waves_sampled(cout):
    """128 -> 128 and 64 -> 64 on [cin, 4, 256, 320]: 1,280 CTA tiles of 16 x 16
    voxels over the 148 SMs (8.6 waves; two accumulators alternate), ragged
    nowhere.  512 sampled voxels (corners, edges, tile and sub-tile seams)
    against the oracle."""
    T, H, W = 4, 256, 320
    x, w, b = synth.conv_input(cin=cout, cout=cout, T=T, H=H, W=W, seed=cout + 3)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    seams = {(t, h, c) for t in (0, 3) for h in (0, 7, 8, 15, 16, 31, 32, 255)
             for c in (0, 15, 16, 319)}
    pts = sorted(set(sample_voxels(T, H, W, 512 - len(seams), seed=8)) | seams)
    got = np.stack([yc[t, h, c].double().numpy() for (t, h, c) in pts], 1)
    ref = np.stack([O.causal_conv3d_at(x, w, b, t, h, c) for (t, h, c) in pts], 1)
    assert_close(got, ref, torch.bfloat16, f"conv {cout} many waves")
    assert torch.isfinite(yc).all()
    assert B.device_error() == 0
