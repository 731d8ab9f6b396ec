"""Guard bands around every buffer a call writes (GPU).

Without a memory checker on these machines, out-of-bounds writes are looked
for directly: each output, workspace and cache a call writes is a view into a
larger byte buffer filled with a sentinel byte, and after the call every byte
outside the view must still hold the sentinel.  The views start 64 KiB into
their buffers, so a stray write before the start is seen as well as one past
the end.  Shapes are ragged (H and W not multiples of the conv tiles, last
tiles partly outside the frame) so that the edge paths of the epilogues run;
each guarded result must also equal the same call on plain buffers bit for bit
(and, for the small cases, the oracle within the bf16 tolerances).
"""
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 64 * 1024
SENT = 0xA5


class Guarded:
    """nbytes of device memory with GUARD sentinel bytes on each side."""

    def __init__(self, nbytes):
        self.n = max(int(nbytes), 16)
        self.buf = torch.full((self.n + 2 * GUARD,), SENT, dtype=torch.uint8, device="cuda")
        self.bytes = self.buf[GUARD:GUARD + self.n]

    def view(self, dtype, shape):
        return self.bytes.view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        for name, part in (("before", self.buf[:GUARD]), ("after", self.buf[GUARD + self.n:])):
            bad = (part != SENT).nonzero()
            assert bad.numel() == 0, (f"{what}: {bad.numel()} guard bytes {name} the buffer changed, "
                                      f"first at offset {int(bad[0])}")


def to_cl(x):
    return x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()


def from_cl(y):
    return y.float().cpu().permute(3, 0, 1, 2).double().numpy()


@pytest.mark.parametrize("C,T,H,W", [(64, 3, 7, 11), (512, 2, 5, 9), (256, 1, 3, 37)])
def test_norm_silu_guarded(C, T, H, W):
    x, g, b = synth.norm_silu_input(C, T, H, W, seed=C)
    xd, gd, bd = to_cl(x), g.cuda(), b.cuda()
    out = Guarded(T * H * W * C * 2)
    y = B.norm_silu(xd, gd, bd, out=out.view(torch.bfloat16, (T, H, W, C)))
    out.check("norm_silu out")
    assert torch.equal(y, B.norm_silu(xd, gd, bd))
    assert_close(from_cl(y), O.norm_silu(x, g, b), torch.bfloat16, "norm_silu guarded")


def _conv_call(xd, pk, out, ws, nws, norm=None, residual=None):
    """wvae_causal_conv3d through the C ABI with the caller's workspace."""
    lib = B.load()
    T, H, W, cin = xd.shape
    kt, kh, kw = pk.k
    g = b = None
    if norm is not None:
        g, b = norm
    B._check("wvae_causal_conv3d", lib.wvae_causal_conv3d(
        B._ptr(xd), None, pk.ptr(), T, H, W, cin, pk.cout, kt, kh, kw, B._ptr(g), B._ptr(b),
        B._ptr(residual), B._ptr(out), B.BF16, B._ptr(ws), nws, B._stream()))
    return out


@pytest.mark.parametrize("cin,cout,T,H,W,with_norm,with_res", [
    (64, 48, 3, 9, 13, False, True),
    (128, 256, 2, 11, 35, True, False),
    (512, 512, 2, 5, 21, True, True),   # CTA pairs (512 output channels)
])
def test_causal_conv3d_guarded(cin, cout, T, H, W, with_norm, with_res):
    x, w, b = synth.conv_input(cin, cout, T, H, W, seed=cin + cout)
    xd = to_cl(x)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    gen = torch.Generator().manual_seed(7)
    norm = None
    if with_norm:
        gm, bt = synth.norm_params(gen, cin)
        norm = (gm.cuda(), bt.cuda())
    res = to_cl(synth.normal(gen, (cout, T, H, W))) if with_res else None
    nws = B.load().wvae_causal_conv3d_workspace_bytes(T, H, W, cin, int(with_norm), B.BF16)
    out = Guarded(T * H * W * cout * 2)
    ws = Guarded(nws)
    y = _conv_call(xd, pk, out.view(torch.bfloat16, (T, H, W, cout)), ws.bytes, nws, norm, res)
    out.check("conv out")
    ws.check("conv workspace")
    assert torch.equal(y, B.causal_conv3d(xd, pk, norm=norm, residual=res))
    assert B.device_error() == 0


@pytest.mark.parametrize("cin,cout", [(64, 128), (128, 128), (256, 128)])
def test_resblock_guarded(cin, cout):
    T, H, W = 2, 9, 21
    x, p = synth.resblock_input(cin, cout, T, H, W, seed=cin)
    blk = B.PackedResBlock(p)
    xd = to_cl(x)
    nws = B.load().wvae_resblock_workspace_bytes(T, H, W, cin, cout, B.BF16)
    out, ws = Guarded(T * H * W * cout * 2), Guarded(nws)
    y = B.resblock(xd, blk, out=out.view(torch.bfloat16, (T, H, W, cout)),
                   workspace=ws.view(torch.uint8, (ws.n,)))
    out.check("resblock out")
    ws.check("resblock workspace")
    assert torch.equal(y, B.resblock(xd, blk))
    assert_close(from_cl(y), O.resblock(x, p), torch.bfloat16, f"resblock {cin}->{cout} guarded")
    assert B.device_error() == 0


@pytest.mark.parametrize("cin,cout,H,W", [(128, 64, 5, 9), (512, 256, 3, 11)])
def test_upsample_conv_guarded(cin, cout, H, W):
    T = 2
    g = torch.Generator().manual_seed(cin)
    x = synth.normal(g, (cin, T, H, W))
    w, b = synth.conv_params(g, cout, cin, 1, 3, 3)
    pk = B.prepack_upsample_conv(w.cuda().bfloat16(), b.cuda())
    xd = to_cl(x)
    lib = B.load()
    nws = lib.wvae_upsample_conv_workspace_bytes(T, H, W, cin, B.BF16)
    out, ws = Guarded(T * 4 * H * W * cout * 2), Guarded(nws)
    y = out.view(torch.bfloat16, (T, 2 * H, 2 * W, cout))
    B._check("wvae_upsample_conv", lib.wvae_upsample_conv(
        B._ptr(xd), B._ptr(y), T, H, W, cin, cout, pk.ptr(), B.BF16, B._ptr(ws.bytes), nws,
        B._stream()))
    out.check("upsample conv out")
    ws.check("upsample conv workspace")
    assert torch.equal(y, B.upsample_conv(xd, pk))
    assert B.device_error() == 0


def test_winograd_conv_guarded():
    cin = cout = 128
    T, H, W = 3, 9, 13
    x, w, b = synth.conv_input(cin, cout, T, H, W, seed=3)
    xd = to_cl(x)
    pw = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
    nws = B.load().wvae_causal_conv3d_winograd_workspace_bytes(T, H, W, cin, cout)
    out, ws = Guarded(T * H * W * cout * 2), Guarded(nws)
    y = B.causal_conv3d_winograd(xd, pw, out=out.view(torch.bfloat16, (T, H, W, cout)),
                                 workspace=ws.view(torch.uint8, (ws.n,)))
    out.check("Winograd conv out")
    ws.check("Winograd conv workspace")
    assert torch.equal(y, B.causal_conv3d_winograd(xd, pw))
    assert B.device_error() == 0


@pytest.mark.parametrize("T,H,W,widths", [
    (2, 3, 5, (128, 128, 64, 64)),
    (3, 12, 20, (64, 64, 64, 128)),   # stage 3: 180 tiles (second tiles per CTA)
    (4, 44, 78, (512, 512, 256, 128)),  # the benchmark's workload
])
def test_decode_trunk_guarded(T, H, W, widths):
    z, params = synth.trunk_input(T=T, H=H, W=W, widths=widths, seed=11)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    shape = (1, 3, T, 16 * H, 16 * W)
    nvid = 3 * T * 256 * H * W * 2
    out, ws = Guarded(nvid), Guarded(tr.workspace_bytes(T, H, W))
    v = B.decode_trunk(zd, tr, out=out.view(torch.bfloat16, shape),
                       workspace=ws.view(torch.uint8, (ws.n,)))
    out.check("trunk video")
    ws.check("trunk workspace")
    assert torch.equal(v, B.decode_trunk(zd, tr))
    assert B.device_error() == 0


def test_video_stream_guarded():
    """The streaming 4T - 3 decode: video, workspace and the causal caches the
    chunks hand on, all guarded; equal to the whole decode."""
    T, H, W = 5, 3, 5
    z, params = synth.trunk_input(T=T, H=H, W=W, widths=(128, 128, 64, 64), seed=13)
    tr = B.PackedTrunk(params)
    zd = z[None].cuda().bfloat16().contiguous()
    stream = B.VideoStream(tr, H, W)
    cache = Guarded(tr.cache_bytes(H, W))
    stream.cache = cache.view(torch.uint8, (cache.n,))
    parts, t0 = [], 0
    for n in (2, 3):
        F = B.video_frames(n, continue_chunk=t0 > 0)
        out = Guarded(3 * F * 256 * H * W * 2)
        ws = Guarded(tr.video_workspace_bytes(n, H, W))
        parts.append(stream.decode(zd[:, :, t0:t0 + n].contiguous(),
                                   out=out.view(torch.bfloat16, (1, 3, F, 16 * H, 16 * W)),
                                   workspace=ws.view(torch.uint8, (ws.n,))))
        out.check(f"video chunk at {t0}")
        ws.check(f"video workspace at {t0}")
        cache.check(f"causal caches after chunk at {t0}")
        t0 += n
    assert torch.equal(torch.cat(parts, 2), B.decode_video(zd, tr))
    assert B.device_error() == 0
