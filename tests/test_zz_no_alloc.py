"""wvae_resblock_noalloc: the residual block for callers that cannot allocate.

Some callers cannot allocate device memory at the point where they run the
block and have no workspace to hand over (a plugin inside a host engine that
owns all device memory, an application that fixes its memory use at start-up).
This entry point takes its scratch from a static 64 MiB array inside the
library instead.  The tests call it through the C ABI:

* twice in a row with different inputs; it runs the same kernels in the same
  launch configuration as wvae_resblock (which uses a caller-provided
  workspace), so each result must equal that one bit for bit, and it is also
  checked against the CPU oracle with the tolerance the other GPU tests use;
* on a shape whose scratch is exactly the 64 MiB limit (after the smaller
  calls, so the array holds an earlier call's data), again bit for bit;
* on a shape that needs 512 bytes more than the limit, which must be rejected
  before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu

WVAE_ERR_WORKSPACE = 4
LIMIT = 64 << 20


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, blk, y, shape=None):
    T, H, W, cin = shape if shape is not None else x.shape
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
        assert torch.equal(y, ref), f"call {call}: differs from wvae_resblock"
        assert_close(from_cl(y), O.resblock(x, p), torch.bfloat16, f"no-alloc call {call}")
    assert B.device_error() == 0


def test_noalloc_at_the_scratch_limit():
    """256 -> 256 on [2, 128, 256]: A1 and A2 take 2 x 65,536 voxels x 256
    channels x 2 bytes = exactly 64 MiB."""
    T, H, W, c = 2, 128, 256, 256
    assert B.load().wvae_resblock_workspace_bytes(T, H, W, c, c, 0) == LIMIT
    x, p = synth.resblock_input(cin=c, cout=c, T=T, H=H, W=W, seed=13)
    blk = B.PackedResBlock(p)
    xd = to_cl(x)
    ref = B.resblock(xd, blk)
    y = torch.full((T, H, W, c), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(xd, blk, y)
    assert st == 0, B.status_string(st)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    assert B.device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """64 -> 64 on [5, 481, 109] (262,145 voxels, an odd count): each of A1 and
    A2 is 33,554,560 bytes, rounded up to 33,554,688, so the block needs
    64 MiB + 512 bytes and must be refused with nothing launched."""
    T, H, W, c = 5, 481, 109, 64
    need = B.load().wvae_resblock_workspace_bytes(T, H, W, c, c, 0)
    assert need == LIMIT + 512
    x, p = synth.resblock_input(cin=c, cout=c, T=1, H=8, W=8, seed=3)
    blk = B.PackedResBlock(p)
    xd = to_cl(x)
    y = torch.zeros((1, 8, 8, c), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(xd, blk, y, shape=(T, H, W, c))
    assert st == WVAE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0          # nothing was launched
    assert np.isfinite(from_cl(xd)).all()
