"""The C-ABI library on the CPU: it loads without a GPU, exports every entry point
include/wvae.h declares, sizes its buffers as documented, and rejects bad
arguments on the host before touching a device."""
import ctypes
import subprocess

import pytest

from video_diffusion_vae_b200 import binding as B

NULL = None
A = ctypes.c_void_p(0x10000)        # a 16-byte aligned fake pointer, never dereferenced
MIS = ctypes.c_void_p(0x10008)      # misaligned fake pointer


@pytest.fixture(scope="module")
def lib():
    return B.load()


def test_exports_every_declared_symbol(lib):
    declared = B.header_symbols()
    assert len(declared) == 33
    out = subprocess.check_output(["nm", "-D", "--defined-only", B.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(lib, s)


def test_status_strings_and_version(lib):
    assert B.status_string(0) == "ok"
    for s in range(1, 8):
        assert B.status_string(s) not in ("ok", "unknown status")
    assert B.status_string(99) == "unknown status"
    assert B.version() >> 16 == 1


def test_packed_bytes(lib):
    # bf16: [cout_pad][taps][cin_pad] bf16, then the fp32 bias at a 256-byte boundary
    n = lib.wvae_conv_packed_bytes(512, 512, 3, 3, 3, B.BF16)
    assert n == 512 * 27 * 512 * 2 + 512 * 4
    n = lib.wvae_conv_packed_bytes(12, 128, 3, 3, 3, B.BF16)   # head: cout padded to 16
    assert n == 16 * 27 * 128 * 2 + 16 * 4
    n = lib.wvae_conv_packed_bytes(512, 48, 3, 3, 3, B.BF16)   # conv_in: cin padded to 64
    assert n == 512 * 27 * 64 * 2 + 512 * 4
    n = lib.wvae_conv_packed_bytes(64, 64, 3, 3, 3, B.F32)
    assert n == 64 * 27 * 64 * 4 + 64 * 4
    assert lib.wvae_conv_packed_bytes(64, 64, 2, 3, 3, B.BF16) == 0      # unsupported kernel
    assert lib.wvae_conv_packed_bytes(0, 64, 3, 3, 3, B.BF16) == 0


def test_workspace_sizes(lib):
    nv = 4 * 176 * 312
    assert lib.wvae_resblock_workspace_bytes(4, 176, 312, 256, 256, B.BF16) == 2 * nv * 256 * 2
    assert lib.wvae_causal_conv3d_workspace_bytes(4, 88, 156, 512, 0, B.BF16) == 0
    assert lib.wvae_causal_conv3d_workspace_bytes(4, 88, 156, 512, 1, B.BF16) == 4 * 88 * 156 * 512 * 2
    assert lib.wvae_upsample_conv_workspace_bytes(4, 88, 156, 512, B.BF16) == 0      # phase convs
    assert lib.wvae_upsample_conv_workspace_bytes(4, 88, 156, 512, B.F32) == 4 * 176 * 312 * 512 * 4
    # four 2x2 phase kernels: [cout_pad][16][cin_pad] bf16 + bias
    assert lib.wvae_upsample_conv_packed_bytes(256, 512, B.BF16) == 256 * 16 * 512 * 2 + 256 * 4
    assert lib.wvae_decode_trunk_workspace_bytes(4, 44, 78, None) > 4 * 352 * 624 * 128 * 4
    assert lib.wvae_decode_trunk_workspace_bytes(0, 44, 78, None) == 0


def test_norm_silu_rejects_on_host(lib):
    s = None
    assert lib.wvae_norm_silu(NULL, A, A, A, 1, 1, 1, 64, 1e-12, B.BF16, s) == 1
    assert lib.wvae_norm_silu(A, A, A, A, 0, 1, 1, 64, 1e-12, B.BF16, s) == 1
    assert lib.wvae_norm_silu(A, A, A, A, 1, 1, 1, 64, 0.0, B.BF16, s) == 1
    assert lib.wvae_norm_silu(A, A, A, A, 1, 1, 1, 60, 1e-12, B.BF16, s) == 2   # C % 8
    assert lib.wvae_norm_silu(A, A, A, A, 1, 1, 1, 2048, 1e-12, B.BF16, s) == 2
    assert lib.wvae_norm_silu(A, A, A, A, 1, 1, 1, 64, 1e-12, 7, s) == 2
    assert lib.wvae_norm_silu(MIS, A, A, A, 1, 1, 1, 64, 1e-12, B.BF16, s) == 3
    # valid arguments but no device in this process
    assert lib.wvae_norm_silu(A, A, A, A, 1, 1, 1, 64, 1e-12, B.BF16, s) == 7


def test_conv_rejects_on_host(lib):
    s = None
    args = lambda **k: dict(dict(x=A, cache=NULL, w=A, T=2, H=4, W=4, cin=64, cout=64, kt=3, kh=3, kw=3,  # noqa: E731
                                 g=NULL, b=NULL, res=NULL, y=ctypes.c_void_p(0x20000), dt=B.BF16,
                                 ws=NULL, nws=0), **k)

    def call(**k):
        a = args(**k)
        return lib.wvae_causal_conv3d(a["x"], a["cache"], a["w"], a["T"], a["H"], a["W"], a["cin"],
                                      a["cout"], a["kt"], a["kh"], a["kw"], a["g"], a["b"], a["res"],
                                      a["y"], a["dt"], a["ws"], a["nws"], s)
    assert call(x=NULL) == 1
    assert call(g=A) == 1                   # gamma without beta
    assert call(y=A) == 1                   # in place
    assert call(kt=2) == 2                  # kernel size
    assert call(cin=48) == 2                # bf16 needs cin % 64
    assert call(cout=24) == 2               # bf16 needs cout % 16
    assert call(cout=384) == 2              # > 256 and != 512
    assert call(x=MIS) == 3
    assert call(g=A, b=A) == 4              # norm needs a workspace
    assert call(cache=A, kt=1, kh=3, kw=3) == 1
    assert call() == 7                      # no device here


def test_resblock_rejects_on_host(lib):
    s = None
    y = ctypes.c_void_p(0x20000)
    f = lib.wvae_resblock
    assert f(A, y, 2, 4, 4, 64, 64, A, A, A, A, A, A, NULL, B.BF16, NULL, 0, s) == 4
    assert f(A, y, 2, 4, 4, 64, 128, A, A, A, A, A, A, NULL, B.BF16, A, 1 << 30, s) == 1  # no shortcut
    assert f(A, y, 2, 4, 4, 64, 64, A, A, A, A, A, A, A, B.BF16, A, 1 << 30, s) == 1     # extra shortcut
    assert f(A, A, 2, 4, 4, 64, 64, A, A, A, A, A, A, NULL, B.BF16, A, 1 << 30, s) == 1   # in place
    assert f(A, y, 2, 4, 4, 64, 64, A, A, A, A, A, A, NULL, B.BF16, A, 1 << 30, s) == 7


def test_trunk_rejects_on_host(lib):
    s = None
    P = (ctypes.c_void_p * 21)(*([0x10000] * 21))
    N = (ctypes.c_void_p * 34)(*([0x10000] * 34))
    y = ctypes.c_void_p(0x20000)
    f = lib.wvae_decode_trunk
    assert f(P, N, A, y, 4, 44, 78, None, B.F32, A, 1 << 40, s) == 2
    bad = (ctypes.c_int * 4)(512, 512, 256, 96)
    assert f(P, N, A, y, 4, 44, 78, bad, B.BF16, A, 1 << 40, s) == 2
    assert f(P, N, A, y, 4, 44, 78, None, B.BF16, A, 16, s) == 4
    P0 = (ctypes.c_void_p * 21)(*([0x10000] * 20 + [0]))
    assert f(P0, N, A, y, 4, 44, 78, None, B.BF16, A, 1 << 40, s) == 1
    assert f(P, N, A, y, 4, 44, 78, None, B.BF16, A, 1 << 40, s) == 7
    assert lib.wvae_decode_trunk_launches() == 22
    E = (ctypes.c_void_p * 44)(*([0x30000] * 44))
    ft = lib.wvae_decode_trunk_timed
    assert ft(P, N, A, y, 4, 44, 78, None, B.BF16, A, 1 << 40, None, 0, s) == 1
    assert ft(P, N, A, y, 4, 44, 78, None, B.BF16, A, 1 << 40, E, 43, s) == 1
    assert ft(P, N, A, y, 4, 44, 78, None, B.BF16, A, 1 << 40, E, 44, s) == 7


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.reload(B)
    try:
        mod._lib = None
        with pytest.raises(RuntimeError, match="libwvae.so not found"):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        importlib.reload(B)


def test_selftest_wait_timeout_rejects_bad_limits():
    """The limit is checked on the host before anything touches a device."""
    lib = B.load()
    for bad in (0, 1000001):
        assert lib.wvae_selftest_wait_timeout(bad, NULL) == 1  # WVAE_ERR_INVALID_ARG


def test_trunk_cache_bytes_and_chunk_validation():
    """The chunked decode's cache holds two input frames of each of the 18
    causal convs; T < 2 and a missing cache are refused on the host."""
    lib = B.load()
    w = (ctypes.c_int * 4)(512, 512, 256, 128)
    H, W = 44, 78
    frames = [H * W * 64] + [(H << s) * (W << s) * c for s, c in enumerate((512, 512, 256, 128))
                             for _ in range(4)] + [(H << 3) * (W << 3) * 128]
    want = sum(-(-2 * f * 2 // 256) * 256 for f in frames)
    assert lib.wvae_decode_trunk_cache_bytes(H, W, w) == want
    assert lib.wvae_decode_trunk_cache_bytes(0, W, w) == 0
    P = (ctypes.c_void_p * 21)(*([A] * 21))
    N = (ctypes.c_void_p * 34)(*([A] * 34))
    # T = 1 cannot hand two frames on; a NULL cache is refused
    assert lib.wvae_decode_trunk_chunk(P, N, A, A, 1, H, W, w, B.BF16, A, 1 << 40, A, 1 << 40, 0,
                                       NULL) == 1
    assert lib.wvae_decode_trunk_chunk(P, N, A, A, 4, H, W, w, B.BF16, A, 1 << 40, NULL, 0, 0,
                                       NULL) == 1



def test_video_decode_frames_and_validation():
    """4T - 3 frames (4T for a continuing chunk); a continuing chunk without a
    cache, T < 2 with a cache, and a short workspace are refused on the host."""
    lib = B.load()
    assert [lib.wvae_decode_video_frames(T, 0) for T in (1, 2, 4, 49)] == [1, 5, 13, 193]
    assert lib.wvae_decode_video_frames(4, 1) == 16 and lib.wvae_decode_video_frames(0, 0) == 0
    w = (ctypes.c_int * 4)(512, 512, 256, 128)
    H, W = 44, 78
    ws = lib.wvae_decode_video_workspace_bytes(4, H, W, w)
    assert ws > lib.wvae_decode_trunk_workspace_bytes(4, H, W, w)
    P = (ctypes.c_void_p * 21)(*([A] * 21))
    N = (ctypes.c_void_p * 34)(*([A] * 34))
    assert lib.wvae_decode_video(P, N, A, A, 4, H, W, w, B.BF16, A, ws, NULL, 0, 1, NULL) == 1
    assert lib.wvae_decode_video(P, N, A, A, 1, H, W, w, B.BF16, A, ws, A, 1 << 40, 0, NULL) == 1
    assert lib.wvae_decode_video(P, N, A, A, 4, H, W, w, B.BF16, A, 1024, NULL, 0, 0, NULL) == 4


def test_winograd_and_row_slab_entry_points_reject_on_host():
    """Refused before any launch: Winograd conv with input channels not a
    multiple of 64, an unsupported output width, aliasing; row-slab steps out
    of range and a slab whose last stage is wider than the head kernel takes."""
    lib = B.load()
    assert lib.wvae_conv_winograd_packed_bytes(64, 64) > lib.wvae_conv_packed_bytes(64, 64, 3, 3, 3, 0)
    ws = lib.wvae_causal_conv3d_winograd_workspace_bytes(2, 9, 17, 64, 64)
    assert ws == 2 * (-(-16 * 2 * 5 * 9 * 64 * 2 // 256) * 256)
    A2 = ctypes.c_void_p(0x20000)
    assert lib.wvae_causal_conv3d_winograd(A, A2, 2, 9, 17, 32, 64, NULL, A2, A, ws, NULL) in (1, 2, 3)
    assert lib.wvae_causal_conv3d_winograd(A, A2, 2, 9, 17, 64, 72, NULL, A2, A, ws, NULL) in (2, 3)
    assert lib.wvae_causal_conv3d_winograd(A, A2, 2, 9, 17, 64, 64, NULL, A, A, ws, NULL) == 1
    w = (ctypes.c_int * 4)(128, 128, 64, 64)
    P = (ctypes.c_void_p * 21)(*([A] * 21))
    N = (ctypes.c_void_p * 34)(*([A] * 34))
    assert lib.wvae_decode_rows_step(22, P, N, A, A, 2, 3, 4, w, B.BF16, A, 1 << 40, NULL) == 1
    assert lib.wvae_decode_rows_step(-1, P, N, A, A, 2, 3, 4, w, B.BF16, A, 1 << 40, NULL) == 1
    off, dims = ctypes.c_size_t(0), (ctypes.c_int * 4)()
    wide = (ctypes.c_int * 4)(128, 128, 64, 256)
    # a last stage wider than the head kernel takes: the whole slab plan is refused
    assert lib.wvae_decode_rows_halo(3, 2, 3, 4, wide, ctypes.byref(off), dims) == 2
    assert lib.wvae_decode_rows_halo(21, 2, 3, 4, wide, ctypes.byref(off), dims) == 2
    assert lib.wvae_decode_rows_halo(3, 2, 3, 4, w, ctypes.byref(off), dims) == 0
