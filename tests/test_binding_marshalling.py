"""The Python binding's argument marshalling on the CPU, against a stand-in of
libwvae.so that takes each call's arguments and checks them against the
parameter list include/wvae.h declares (count, pointer / integer / size kind).

Only the device check of the binding is relaxed (CPU tensors stand in for CUDA
ones); every other check and every call runs as on the GPU, so a binding that
passes an argument too many, too few or of the wrong kind fails here."""
import ctypes
import re

import pytest
import torch

from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth


def header_params():
    """{function: [parameter declaration, ...]} from include/wvae.h."""
    txt = open(B.HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    out = {}
    for m in re.finditer(r"^WVAE_API\s+[\w\s\*]*?\b(wvae_\w+)\s*\(([^)]*)\)", txt, flags=re.M):
        ps = " ".join(m.group(2).split())
        out[m.group(1)] = [] if ps in ("", "void") else [p.strip() for p in ps.split(",")]
    return out


def kind(decl):
    if "*" in decl or decl.split()[0] == "wvae_stream_t":
        return "ptr"
    if decl.split()[0] == "float":
        return "float"
    return "int"


class FakeLib:
    """Stands in for libwvae.so: checks every call against the header, records it."""

    def __init__(self):
        self.params = header_params()
        self.calls = []

    def __getattr__(self, name):
        if name not in self.params:
            raise AttributeError(name)
        decls = self.params[name]

        def call(*args):
            assert len(args) == len(decls), f"{name}: {len(args)} arguments, header declares {len(decls)}"
            for a, d in zip(args, decls):
                k = kind(d)
                if k == "ptr":
                    assert a is None or isinstance(a, (ctypes.c_void_p, ctypes.Array, ctypes._Pointer)), \
                        f"{name}: {d} got {type(a).__name__}"
                elif k == "float":
                    assert isinstance(a, float), f"{name}: {d} got {type(a).__name__}"
                else:
                    assert isinstance(a, int) and not isinstance(a, bool), f"{name}: {d} got {type(a).__name__}"
            self.calls.append((name, args))
            if name.endswith("_bytes"):
                return 4096
            if name == "wvae_decode_trunk_launches":
                return 22
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    real_cuda = B._cuda

    def cpu_ok(t, name, dtype=None, shape=None):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        return t

    monkeypatch.setattr(B, "load", lambda path=None: lib)
    monkeypatch.setattr(B, "_stream", lambda: ctypes.c_void_p(0))
    monkeypatch.setattr(B, "_cuda", cpu_ok)
    lib.real_cuda = real_cuda
    return lib


def names(lib):
    return [c[0] for c in lib.calls]


def test_every_header_function_has_a_parameter_list():
    ps = header_params()
    assert set(ps) == set(B.header_symbols())
    assert len(ps["wvae_causal_conv3d"]) == 19 and len(ps["wvae_decode_trunk_chunk"]) == 15


def test_norm_conv_resblock_upsample(fake):
    x, g, b = synth.norm_silu_input(C=64, T=1, H=2, W=3)
    xl = x.permute(1, 2, 3, 0).contiguous().bfloat16()
    y = B.norm_silu(xl, g, b)
    assert y.shape == xl.shape and names(fake)[-1] == "wvae_norm_silu"

    xc, p = synth.tiny_resblock(bf16=True, c=64, T=2, H=4, W=4)
    xcl = xc.permute(1, 2, 3, 0).contiguous().bfloat16()
    blk = B.PackedResBlock(p, torch.bfloat16, device="cpu")
    assert blk.w1.blob.numel() == 4096               # the size the library reported
    B.causal_conv3d(xcl, blk.w1, norm=(blk.gamma1, blk.beta1), residual=xcl)
    assert names(fake)[-2:] == ["wvae_causal_conv3d_workspace_bytes", "wvae_causal_conv3d"]
    B.resblock(xcl, blk)
    B.resblock(xcl, blk, workspace=torch.empty(100, dtype=torch.float32))
    ws_arg = fake.calls[-1][1][16]
    assert fake.calls[-1][0] == "wvae_resblock" and ws_arg == 400  # bytes, not elements

    wu = torch.randn(32, 64, 1, 3, 3).bfloat16()
    pu = B.prepack_upsample_conv(wu, torch.zeros(32))
    yu = B.upsample_conv(xcl, pu)
    assert yu.shape == (2, 8, 8, 32) and names(fake)[-1] == "wvae_upsample_conv"


def test_trunk_and_stream(fake):
    z, params = synth.trunk_input(T=2, H=2, W=3, widths=(64, 64, 64, 64), blocks=2)
    tr = B.PackedTrunk(params, device="cpu")
    assert len(tr.convs) == B.TRUNK_PACKED
    zd = z[None].bfloat16().contiguous()
    v = B.decode_trunk(zd, tr)
    assert v.shape == (1, 3, 2, 32, 48) and names(fake)[-1] == "wvae_decode_trunk"
    st = B.TrunkStream(tr, 2, 3, device="cpu")
    st.decode(zd)
    st.decode(zd)
    chunk_calls = [c for c in fake.calls if c[0] == "wvae_decode_trunk_chunk"]
    assert [c[1][13] for c in chunk_calls] == [0, 1]   # continue_chunk: first chunk, then carried


def test_video_decode_and_stream(fake):
    """The temporal decode: 4T - 3 frames for a whole decode or a first chunk,
    4T for a continuing one; no cache for a whole decode."""
    fake.wvae_decode_video_frames = lambda T, c: 4 * T if c else 4 * T - 3
    z, params = synth.trunk_input(T=2, H=2, W=3, widths=(64, 64, 64, 64), blocks=2)
    tr = B.PackedTrunk(params, device="cpu")
    zd = z[None].bfloat16().contiguous()
    v = B.decode_video(zd, tr)
    assert v.shape == (1, 3, 5, 32, 48) and names(fake)[-1] == "wvae_decode_video"
    assert fake.calls[-1][1][11] is None and fake.calls[-1][1][13] == 0   # cache, continue
    st = B.VideoStream(tr, 2, 3, device="cpu")
    a, b = st.decode(zd), st.decode(zd)
    assert a.shape[2] == 5 and b.shape[2] == 8
    calls = [c for c in fake.calls if c[0] == "wvae_decode_video"]
    assert [c[1][13] for c in calls] == [0, 0, 1]


def test_caller_workspace_must_be_a_cuda_tensor(fake):
    with pytest.raises(TypeError):
        fake.real_cuda(torch.empty(64, dtype=torch.uint8), "workspace")
    with pytest.raises(TypeError):
        B._ws([0] * 64, 64, "cpu")
