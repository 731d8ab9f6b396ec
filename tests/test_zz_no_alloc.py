"""wvae_resblock_noalloc: the residual block for callers that cannot allocate.

Some callers cannot allocate device memory at the point where they run the
block and have no workspace to hand over (a plugin inside a host engine that
owns all device memory, an application that fixes its memory use at start-up).
This entry point takes its scratch from a static 64 MiB array inside the
library instead.  The test calls it through the C ABI, twice in a row with
different inputs, and checks each result against wvae_resblock (which uses a
caller-provided workspace) with the tolerance the other GPU tests use.  It also
checks that a shape whose scratch would not fit is rejected before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import assert_close, from_cl, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu

WVAE_ERR_WORKSPACE = 4


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, blk, y):
    T, H, W, cin = x.shape
    lib = B.load()
    return lib.wvae_resblock_noalloc(
        _ptr(x), _ptr(y), T, H, W, cin, blk.cout, _ptr(blk.gamma1), _ptr(blk.beta1), blk.w1.ptr(),
        _ptr(blk.gamma2), _ptr(blk.beta2), blk.w2.ptr(), None if blk.ws is None else blk.ws.ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("cin,cout,T,H,W", [(256, 256, 2, 40, 72), (256, 128, 3, 21, 37)])
def test_noalloc_matches_resblock_two_calls(cin, cout, T, H, W):
    for call, seed in enumerate((11, 12)):
        x, p = synth.resblock_input(cin=cin, cout=cout, T=T, H=H, W=W, seed=seed)
        blk = B.PackedResBlock(p)
        xd = to_cl(x)
        ref = B.resblock(xd, blk)
        y = torch.full((T, H, W, cout), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _noalloc(xd, blk, y)
        assert st == 0, f"call {call}: {B.status_string(st)}"
        torch.cuda.synchronize()
        assert_close(from_cl(y), from_cl(ref), torch.bfloat16, f"no-alloc call {call}")
    assert B.device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    x, p = synth.resblock_input(cin=256, cout=256, T=1, H=8, W=8, seed=3)
    blk = B.PackedResBlock(p)
    xd = to_cl(x)
    y = torch.zeros((1, 8, 8, 256), dtype=torch.bfloat16, device="cuda")
    lib = B.load()
    # [4, 176, 312] x (256 + 256) channels x 2 bytes = 225 MB > 64 MiB
    st = lib.wvae_resblock_noalloc(
        _ptr(xd), _ptr(y), 4, 176, 312, 256, 256, _ptr(blk.gamma1), _ptr(blk.beta1), blk.w1.ptr(),
        _ptr(blk.gamma2), _ptr(blk.beta2), blk.w2.ptr(), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == WVAE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0          # nothing was launched
    assert np.isfinite(from_cl(xd)).all()
