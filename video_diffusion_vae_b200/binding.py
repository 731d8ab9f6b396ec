"""Python binding of libwvae.so (include/wvae.h): argument marshalling only.

Every function takes torch CUDA tensors, checks dtype/shape/contiguity, hands
their device pointers and the current stream to the C ABI and raises
:class:`WvaeError` on a non-zero status.  Outputs and workspaces are allocated
here with torch (the library itself never allocates).  Activations are
channels-last ``[T, H, W, C]`` (batch 1); the trunk takes NCDHW latents and
returns the NCDHW video.

There is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwvae.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "wvae.h")

BF16, F32 = 0, 1
OK = 0
TRUNK_PACKED = 21
TRUNK_NORMS = 34
DEFAULT_WIDTHS = (512, 512, 256, 128)

_lib = None
_lock = threading.Lock()


class WvaeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def load(path: str | None = None):
    """Load libwvae.so (built in-tree by video_diffusion_vae_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libwvae.so not found at {p}: run `python -m video_diffusion_vae_b200.build`")
        lib = ctypes.CDLL(p)
        V, S, I, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        sig = {
            "wvae_status_string": (ctypes.c_char_p, [I]),
            "wvae_version": (I, []),
            "wvae_device_error": (I, [ctypes.POINTER(ctypes.c_uint), I]),
            "wvae_selftest_wait_timeout": (I, [ctypes.c_uint, V]),
            "wvae_norm_silu": (I, [V, V, V, V, I, I, I, I, F, I, V]),
            "wvae_conv_packed_bytes": (S, [I, I, I, I, I, I]),
            "wvae_prepack_conv": (I, [V, I, V, I, I, I, I, I, I, V, S, V]),
            "wvae_causal_conv3d_workspace_bytes": (S, [I, I, I, I, I, I]),
            "wvae_causal_conv3d": (I, [V, V, V, I, I, I, I, I, I, I, I, V, V, V, V, I, V, S, V]),
            "wvae_resblock_workspace_bytes": (S, [I, I, I, I, I, I]),
            "wvae_resblock": (I, [V, V, I, I, I, I, I, V, V, V, V, V, V, V, I, V, S, V]),
            "wvae_upsample_conv_packed_bytes": (S, [I, I, I]),
            "wvae_prepack_upsample_conv": (I, [V, I, V, I, I, I, V, S, V]),
            "wvae_upsample_conv_workspace_bytes": (S, [I, I, I, I, I]),
            "wvae_upsample_conv": (I, [V, V, I, I, I, I, I, V, I, V, S, V]),
            "wvae_decode_trunk_workspace_bytes": (S, [I, I, I, ctypes.POINTER(I)]),
            "wvae_decode_trunk": (I, [ctypes.POINTER(V), ctypes.POINTER(V), V, V, I, I, I,
                                      ctypes.POINTER(I), I, V, S, V]),
            "wvae_decode_trunk_launches": (I, []),
            "wvae_resblock_noalloc": (I, [V, V, I, I, I, I, I, V, V, V, V, V, V, V, V]),
            "wvae_decode_trunk_timed": (I, [ctypes.POINTER(V), ctypes.POINTER(V), V, V, I, I, I,
                                            ctypes.POINTER(I), I, V, S, ctypes.POINTER(V), I, V]),
            "wvae_decode_trunk_cache_bytes": (S, [I, I, ctypes.POINTER(I)]),
            "wvae_decode_trunk_chunk": (I, [ctypes.POINTER(V), ctypes.POINTER(V), V, V, I, I, I,
                                            ctypes.POINTER(I), I, V, S, V, S, I, V]),
            "wvae_conv_winograd_packed_bytes": (S, [I, I]),
            "wvae_prepack_conv_winograd": (I, [V, I, V, I, I, V, S, V]),
            "wvae_causal_conv3d_winograd_workspace_bytes": (S, [I, I, I, I, I]),
            "wvae_causal_conv3d_winograd": (I, [V, V, I, I, I, I, I, V, V, V, S, V]),
            "wvae_decode_rows_steps": (I, []),
            "wvae_decode_rows_workspace_bytes": (S, [I, I, I, ctypes.POINTER(I)]),
            "wvae_decode_rows_halo": (I, [I, I, I, I, ctypes.POINTER(I), ctypes.POINTER(S),
                                          ctypes.POINTER(I)]),
            "wvae_decode_rows_step": (I, [I, ctypes.POINTER(V), ctypes.POINTER(V), V, V, I, I, I,
                                          ctypes.POINTER(I), I, V, S, V]),
            "wvae_decode_video_frames": (I, [I, I]),
            "wvae_decode_video_workspace_bytes": (S, [I, I, I, ctypes.POINTER(I)]),
            "wvae_decode_video": (I, [ctypes.POINTER(V), ctypes.POINTER(V), V, V, I, I, I,
                                      ctypes.POINTER(I), I, V, S, V, S, I, V]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
        return lib


def header_symbols(header: str = HEADER):
    """Names of the entry points declared in include/wvae.h."""
    txt = open(header).read()
    return sorted(set(re.findall(r"^WVAE_API\s+[\w\s\*]*?\b(wvae_\w+)\s*\(", txt, flags=re.M)))


def status_string(status: int) -> str:
    return load().wvae_status_string(int(status)).decode()


def _check(fn, status):
    if status != OK:
        raise WvaeError(fn, status)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _f32vec(t, n, name):
    return _cuda(t, name, torch.float32, (n,))


def _workspace(nbytes, device):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def _nbytes(t):
    return t.numel() * t.element_size()


def _ws(workspace, nbytes, device):
    """The caller's workspace (a contiguous CUDA tensor of any dtype: its size in
    bytes goes to the library, which rejects one that is too small), else a new
    one of nbytes on device."""
    if workspace is None:
        return _workspace(nbytes, device)
    return _cuda(workspace, "workspace")


def version() -> int:
    return load().wvae_version()


def device_error(reset: bool = True) -> int:
    """Raw device error word (0 = no kernel recorded a fault); synchronises."""
    code = ctypes.c_uint(0)
    st = load().wvae_device_error(ctypes.byref(code), int(reset))
    if st not in (OK, 6):
        raise WvaeError("wvae_device_error", st)
    return code.value


def selftest_wait_timeout(limit_us: int = 20000):
    """Enqueue the bounded-wait self-test (a wait that nothing completes gives
    up after limit_us and sets bit 0x10 of the device error word)."""
    _check("wvae_selftest_wait_timeout", load().wvae_selftest_wait_timeout(int(limit_us), _stream()))


# ------------------------------------------------------------------ norm-SiLU
def norm_silu(x, gamma, beta, eps: float = 1e-12, out=None):
    """SiLU(x / max(||x||_2 over C, eps) * sqrt(C) * gamma + beta); x [T, H, W, C]."""
    _cuda(x, "x")
    T, H, W, C = x.shape
    y = torch.empty_like(x) if out is None else _cuda(out, "out", x.dtype, x.shape)
    _check("wvae_norm_silu", load().wvae_norm_silu(
        _ptr(x), _ptr(y), _ptr(_f32vec(gamma, C, "gamma")), _ptr(_f32vec(beta, C, "beta")),
        T, H, W, C, float(eps), _dt(x), _stream()))
    return y


# -------------------------------------------------------------------- prepack
class PackedConv:
    """A conv's weights in the kernel tile order (device bytes) plus its shape."""

    def __init__(self, blob, cout, cin, k, dtype):
        self.blob, self.cout, self.cin, self.k, self.dtype = blob, cout, cin, tuple(k), dtype

    def ptr(self):
        return ctypes.c_void_p(self.blob.data_ptr())


def prepack_conv(w, bias=None, dtype=torch.bfloat16) -> PackedConv:
    """w: PyTorch [Cout, Cin, KT, KH, KW] (fp32 or bf16, CUDA); bias fp32 [Cout] or None."""
    _cuda(w, "w")
    cout, cin, kt, kh, kw = w.shape
    dt = BF16 if dtype == torch.bfloat16 else F32
    n = load().wvae_conv_packed_bytes(cout, cin, kt, kh, kw, dt)
    if n == 0:
        raise ValueError(f"unsupported conv shape {tuple(w.shape)}")
    blob = torch.empty(n, dtype=torch.uint8, device=w.device)
    b = None if bias is None else _f32vec(bias, cout, "bias")
    _check("wvae_prepack_conv", load().wvae_prepack_conv(
        _ptr(w), _dt(w), _ptr(b), cout, cin, kt, kh, kw, dt, _ptr(blob), n, _stream()))
    return PackedConv(blob, cout, cin, (kt, kh, kw), dt)


def prepack_upsample_conv(w, bias=None, dtype=torch.bfloat16) -> PackedConv:
    """Upsample-conv weights [Cout, Cin, 1, 3, 3] -> the four 2x2 phase kernels (bf16)
    or the plain fp32 packing (fp32 reference path)."""
    _cuda(w, "w")
    cout, cin, kt, kh, kw = w.shape
    if (kt, kh, kw) != (1, 3, 3):
        raise ValueError("upsample conv weights must be [Cout, Cin, 1, 3, 3]")
    dt = BF16 if dtype == torch.bfloat16 else F32
    n = load().wvae_upsample_conv_packed_bytes(cout, cin, dt)
    blob = torch.empty(n, dtype=torch.uint8, device=w.device)
    b = None if bias is None else _f32vec(bias, cout, "bias")
    _check("wvae_prepack_upsample_conv", load().wvae_prepack_upsample_conv(
        _ptr(w), _dt(w), _ptr(b), cout, cin, dt, _ptr(blob), n, _stream()))
    return PackedConv(blob, cout, cin, (1, 3, 3), dt)


# ---------------------------------------------------------------- causal conv
def causal_conv3d(x, packed: PackedConv, cache=None, norm=None, residual=None, out=None):
    """Causal conv of x [T, H, W, Cin]; norm = (gamma, beta) applies SiLU(norm(x)) first."""
    _cuda(x, "x")
    T, H, W, cin = x.shape
    cout = packed.cout
    kt, kh, kw = packed.k
    dt = _dt(x)
    y = torch.empty((T, H, W, cout), dtype=x.dtype, device=x.device) if out is None else \
        _cuda(out, "out", x.dtype, (T, H, W, cout))
    if cache is not None:
        _cuda(cache, "cache", x.dtype, (kt - 1, H, W, cin))
    if residual is not None:
        _cuda(residual, "residual", x.dtype, (T, H, W, cout))
    g = b = None
    if norm is not None:
        g, b = _f32vec(norm[0], cin, "gamma"), _f32vec(norm[1], cin, "beta")
    lib = load()
    nws = lib.wvae_causal_conv3d_workspace_bytes(T, H, W, cin, int(norm is not None), dt)
    ws = _workspace(nws, x.device) if nws else None
    _check("wvae_causal_conv3d", lib.wvae_causal_conv3d(
        _ptr(x), _ptr(cache), packed.ptr(), T, H, W, cin, cout, kt, kh, kw, _ptr(g), _ptr(b),
        _ptr(residual), _ptr(y), dt, _ptr(ws), nws, _stream()))
    return y


# ------------------------------------------------ causal conv, Winograd form
def prepack_conv_winograd(w, bias=None) -> PackedConv:
    """w: PyTorch [Cout, Cin, 3, 3, 3] (fp32 or bf16, CUDA) -> the Winograd-transformed
    weights (fp16) for causal_conv3d_winograd."""
    _cuda(w, "w")
    cout, cin, kt, kh, kw = w.shape
    if (kt, kh, kw) != (3, 3, 3):
        raise ValueError("Winograd weights must be [Cout, Cin, 3, 3, 3]")
    n = load().wvae_conv_winograd_packed_bytes(cout, cin)
    blob = torch.empty(n, dtype=torch.uint8, device=w.device)
    b = None if bias is None else _f32vec(bias, cout, "bias")
    _check("wvae_prepack_conv_winograd", load().wvae_prepack_conv_winograd(
        _ptr(w), _dt(w), _ptr(b), cout, cin, _ptr(blob), n, _stream()))
    return PackedConv(blob, cout, cin, (3, 3, 3), BF16)


def causal_conv3d_winograd(x, packed: PackedConv, residual=None, out=None, workspace=None):
    """The causal 3x3x3 conv of x [T, H, W, Cin] bf16 as Winograd F(2x2, 3x3) products."""
    _cuda(x, "x", torch.bfloat16)
    T, H, W, cin = x.shape
    cout = packed.cout
    y = torch.empty((T, H, W, cout), dtype=x.dtype, device=x.device) if out is None else \
        _cuda(out, "out", x.dtype, (T, H, W, cout))
    if residual is not None:
        _cuda(residual, "residual", x.dtype, (T, H, W, cout))
    lib = load()
    ws = _ws(workspace, lib.wvae_causal_conv3d_winograd_workspace_bytes(T, H, W, cin, cout), x.device)
    _check("wvae_causal_conv3d_winograd", lib.wvae_causal_conv3d_winograd(
        _ptr(x), packed.ptr(), T, H, W, cin, cout, _ptr(residual), _ptr(y), _ptr(ws), _nbytes(ws),
        _stream()))
    return y


# ------------------------------------------------------------- residual block
class PackedResBlock:
    def __init__(self, p, dtype=torch.bfloat16, device="cuda"):
        """p: the synth.resblock_params dict (CPU tensors)."""
        wdt = dtype
        self.cin = p["w1"].shape[1]
        self.cout = p["w1"].shape[0]
        dev = torch.device(device)
        f = lambda t: t.to(dev, torch.float32).contiguous()  # noqa: E731
        self.gamma1, self.beta1 = f(p["gamma1"]), f(p["beta1"])
        self.gamma2, self.beta2 = f(p["gamma2"]), f(p["beta2"])
        self.w1 = prepack_conv(p["w1"].to(dev, wdt).contiguous(), f(p["b1"]), dtype)
        self.w2 = prepack_conv(p["w2"].to(dev, wdt).contiguous(), f(p["b2"]), dtype)
        self.ws = prepack_conv(p["ws"].to(dev, wdt).contiguous(), f(p["bs"]), dtype) \
            if p.get("ws") is not None else None


def resblock(x, blk: PackedResBlock, out=None, workspace=None):
    _cuda(x, "x")
    T, H, W, cin = x.shape
    cout = blk.cout
    dt = _dt(x)
    y = torch.empty((T, H, W, cout), dtype=x.dtype, device=x.device) if out is None else \
        _cuda(out, "out", x.dtype, (T, H, W, cout))
    lib = load()
    nws = lib.wvae_resblock_workspace_bytes(T, H, W, cin, cout, dt)
    ws = _ws(workspace, nws, x.device)
    _check("wvae_resblock", lib.wvae_resblock(
        _ptr(x), _ptr(y), T, H, W, cin, cout, _ptr(blk.gamma1), _ptr(blk.beta1), blk.w1.ptr(),
        _ptr(blk.gamma2), _ptr(blk.beta2), blk.w2.ptr(), None if blk.ws is None else blk.ws.ptr(),
        dt, _ptr(ws), _nbytes(ws), _stream()))
    return y


# ------------------------------------------------------- upsample + 3x3 conv
def upsample_conv(x, packed: PackedConv, out=None):
    _cuda(x, "x")
    T, H, W, cin = x.shape
    cout = packed.cout
    dt = _dt(x)
    y = torch.empty((T, 2 * H, 2 * W, cout), dtype=x.dtype, device=x.device) if out is None else \
        _cuda(out, "out", x.dtype, (T, 2 * H, 2 * W, cout))
    lib = load()
    nws = lib.wvae_upsample_conv_workspace_bytes(T, H, W, cin, dt)
    ws = _workspace(nws, x.device) if nws else None
    _check("wvae_upsample_conv", lib.wvae_upsample_conv(
        _ptr(x), _ptr(y), T, H, W, cin, cout, packed.ptr(), dt, _ptr(ws), nws, _stream()))
    return y


# ---------------------------------------------------------------- decoder trunk
class PackedTrunk:
    """All 21 convs prepacked (bf16) and the 17 norms' gamma/beta, in forward order."""

    def __init__(self, params, device="cuda"):
        dev = torch.device(device)
        f = lambda t: t.to(dev, torch.float32).contiguous()  # noqa: E731
        pk = lambda w, b: prepack_conv(w.to(dev, torch.bfloat16).contiguous(), f(b))  # noqa: E731
        self.convs, self.norms = [], []
        self.widths = tuple(int(st["blocks"][0]["w1"].shape[0]) for st in params["stages"])
        self.convs.append(pk(*params["conv_in"]))
        for st in params["stages"]:
            for bp in st["blocks"]:
                self.norms += [f(bp["gamma1"]), f(bp["beta1"]), f(bp["gamma2"]), f(bp["beta2"])]
                self.convs += [pk(bp["w1"], bp["b1"]), pk(bp["w2"], bp["b2"])]
            if st["up"] is not None:
                wu, bu = st["up"]
                self.convs.append(prepack_upsample_conv(wu.to(dev, torch.bfloat16).contiguous(), f(bu)))
        hp = params["head"]
        self.norms += [f(hp["gamma"]), f(hp["beta"])]
        self.convs.append(pk(hp["w"], hp["b"]))
        assert len(self.convs) == TRUNK_PACKED and len(self.norms) == TRUNK_NORMS
        V = ctypes.c_void_p
        self._packed_arr = (V * TRUNK_PACKED)(*[c.blob.data_ptr() for c in self.convs])
        self._norm_arr = (V * TRUNK_NORMS)(*[t.data_ptr() for t in self.norms])
        self._widths_arr = (ctypes.c_int * 4)(*self.widths)

    def workspace_bytes(self, T, H, W):
        return load().wvae_decode_trunk_workspace_bytes(T, H, W, self._widths_arr)

    def cache_bytes(self, H, W):
        return load().wvae_decode_trunk_cache_bytes(H, W, self._widths_arr)

    def video_workspace_bytes(self, T, H, W):
        return load().wvae_decode_video_workspace_bytes(T, H, W, self._widths_arr)


def trunk_launches() -> int:
    return load().wvae_decode_trunk_launches()


def decode_trunk(z, trunk: PackedTrunk, out=None, workspace=None, events=None):
    """z: latents [1, 48, T, H, W] bf16 (CUDA) -> video [1, 3, T, 16H, 16W] bf16.

    events: optional list of 2 * trunk_launches() torch.cuda.Event(enable_timing=True);
    events[2i] / events[2i+1] are recorded around the trunk's i-th kernel launch."""
    _cuda(z, "z", torch.bfloat16)
    _, zc, T, H, W = z.shape
    if zc != 48 or z.shape[0] != 1:
        raise ValueError("z must be [1, 48, T, H, W]")
    y = torch.empty((1, 3, T, 16 * H, 16 * W), dtype=torch.bfloat16, device=z.device) if out is None \
        else _cuda(out, "out", torch.bfloat16, (1, 3, T, 16 * H, 16 * W))
    ws = _ws(workspace, trunk.workspace_bytes(T, H, W), z.device)
    if events is None:
        _check("wvae_decode_trunk", load().wvae_decode_trunk(
            trunk._packed_arr, trunk._norm_arr, _ptr(z), _ptr(y), T, H, W, trunk._widths_arr, BF16,
            _ptr(ws), _nbytes(ws), _stream()))
        return y
    handles = []
    for ev in events:
        if not ev.cuda_event:
            ev.record()          # creates the underlying cudaEvent_t
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _check("wvae_decode_trunk_timed", load().wvae_decode_trunk_timed(
        trunk._packed_arr, trunk._norm_arr, _ptr(z), _ptr(y), T, H, W, trunk._widths_arr, BF16,
        _ptr(ws), _nbytes(ws), arr, len(handles), _stream()))
    return y


class TrunkStream:
    """Chunked decode with the causal caches carried between chunks: feeding the
    latents chunk by chunk gives the video of decoding them at once."""

    def __init__(self, trunk: PackedTrunk, H, W, device="cuda"):
        self.trunk, self.H, self.W = trunk, H, W
        self.cache = _workspace(trunk.cache_bytes(H, W), torch.device(device))
        self.started = False

    def decode(self, z, out=None, workspace=None):
        """z: the next chunk of latents [1, 48, T, H, W] bf16 (T >= 2) -> its video."""
        _cuda(z, "z", torch.bfloat16)
        _, zc, T, H, W = z.shape
        if zc != 48 or z.shape[0] != 1 or (H, W) != (self.H, self.W):
            raise ValueError(f"z must be [1, 48, T, {self.H}, {self.W}]")
        y = torch.empty((1, 3, T, 16 * H, 16 * W), dtype=torch.bfloat16, device=z.device) \
            if out is None else _cuda(out, "out", torch.bfloat16, (1, 3, T, 16 * H, 16 * W))
        tr = self.trunk
        ws = _ws(workspace, tr.workspace_bytes(T, H, W), z.device)
        _check("wvae_decode_trunk_chunk", load().wvae_decode_trunk_chunk(
            tr._packed_arr, tr._norm_arr, _ptr(z), _ptr(y), T, H, W, tr._widths_arr, BF16,
            _ptr(ws), _nbytes(ws), _ptr(self.cache), _nbytes(self.cache), int(self.started),
            _stream()))
        self.started = True
        return y



def video_frames(T: int, continue_chunk: bool = False) -> int:
    """Video frames of a decode with temporal upsampling: 4T - 3, or 4T for a
    continuing chunk."""
    return load().wvae_decode_video_frames(int(T), int(continue_chunk))


def _decode_video(z, trunk, out, workspace, cache, started):
    _cuda(z, "z", torch.bfloat16)
    _, zc, T, H, W = z.shape
    if zc != 48 or z.shape[0] != 1:
        raise ValueError("z must be [1, 48, T, H, W]")
    n = video_frames(T, started)
    y = torch.empty((1, 3, n, 16 * H, 16 * W), dtype=torch.bfloat16, device=z.device) \
        if out is None else _cuda(out, "out", torch.bfloat16, (1, 3, n, 16 * H, 16 * W))
    ws = _ws(workspace, trunk.video_workspace_bytes(T, H, W), z.device)
    _check("wvae_decode_video", load().wvae_decode_video(
        trunk._packed_arr, trunk._norm_arr, _ptr(z), _ptr(y), T, H, W, trunk._widths_arr, BF16,
        _ptr(ws), _nbytes(ws), _ptr(cache), 0 if cache is None else _nbytes(cache), int(started),
        _stream()))
    return y


def decode_video(z, trunk: PackedTrunk, out=None, workspace=None):
    """z: latents [1, 48, T, H, W] bf16 (CUDA) -> video [1, 3, 4T - 3, 16H, 16W] bf16:
    the trunk with the temporal 2x steps after the first two upsample convs."""
    return _decode_video(z, trunk, out, workspace, None, False)


class VideoStream:
    """Chunked decode with temporal upsampling: the first chunk of T latent
    frames gives 4T - 3 video frames, each later one 4T; concatenated, they
    equal decode_video of all the latents."""

    def __init__(self, trunk: PackedTrunk, H, W, device="cuda"):
        self.trunk, self.H, self.W = trunk, H, W
        self.cache = _workspace(trunk.cache_bytes(H, W), torch.device(device))
        self.started = False

    def decode(self, z, out=None, workspace=None):
        if tuple(z.shape[3:]) != (self.H, self.W):
            raise ValueError(f"z must be [1, 48, T, {self.H}, {self.W}]")
        y = _decode_video(z, self.trunk, out, workspace, self.cache, self.started)
        self.started = True
        return y


class RowSlab:
    """One rank's part of a decode split by latent rows (wvae_decode_rows_*):
    its workspace, and for every launch the view of the tensor whose halo rows
    must be filled before it (None when the launch needs no exchange)."""

    def __init__(self, trunk: PackedTrunk, T, rows, W, device="cuda"):
        lib = load()
        self.trunk, self.T, self.rows, self.W = trunk, T, rows, W
        self.steps = lib.wvae_decode_rows_steps()
        n = lib.wvae_decode_rows_workspace_bytes(T, rows, W, trunk._widths_arr)
        if n == 0:
            raise ValueError("unsupported row slab")
        self.ws = _workspace(n, torch.device(device))
        self.halo = []
        for i in range(self.steps):
            off = ctypes.c_size_t(0)
            dims = (ctypes.c_int * 4)()
            _check("wvae_decode_rows_halo", lib.wvae_decode_rows_halo(
                i, T, rows, W, trunk._widths_arr, ctypes.byref(off), dims))
            if dims[0] == 0:
                self.halo.append(None)
                continue
            nel = dims[0] * dims[1] * dims[2] * dims[3]
            flat = self.ws[off.value:off.value + 2 * nel].view(torch.bfloat16)
            self.halo.append(flat.view(dims[0], dims[1], dims[2], dims[3]))

    def step(self, i, z_rows, video_rows):
        """Enqueue launch i (z_rows [1, 48, T, rows + 2, W], video_rows [1, 3, T, 16 rows, 16 W])."""
        tr = self.trunk
        _check("wvae_decode_rows_step", load().wvae_decode_rows_step(
            i, tr._packed_arr, tr._norm_arr, _ptr(z_rows), _ptr(video_rows), self.T, self.rows,
            self.W, tr._widths_arr, BF16, _ptr(self.ws), _nbytes(self.ws), _stream()))


class TrunkGraph:
    """One trunk decode captured as a CUDA graph on fixed buffers: replay()
    re-runs its 22 launches with a single host call (copy the next latents into
    `.z` first).  The library's host work (tensor-map encoding, launch
    configuration) happens once, at capture."""

    def __init__(self, trunk: PackedTrunk, z):
        _cuda(z, "z", torch.bfloat16)
        self.z = z
        _, _, T, H, W = z.shape
        self.out = torch.empty((1, 3, T, 16 * H, 16 * W), dtype=torch.bfloat16, device=z.device)
        self.ws = _workspace(trunk.workspace_bytes(T, H, W), z.device)
        decode_trunk(self.z, trunk, out=self.out, workspace=self.ws)  # device set-up, kernel attributes
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            decode_trunk(self.z, trunk, out=self.out, workspace=self.ws)

    def replay(self):
        self.graph.replay()
        return self.out
