"""Failure detection on the GPU without a fault: a pipeline wait that nothing
completes runs out after a short limit, the kernel records its bit in the
device error word and returns, and the context stays usable."""
import time

import pytest
import torch

from oracle import oracle as O
from tests.gpu_util import assert_close, from_cl, to_cl
from video_diffusion_vae_b200 import binding as B
from video_diffusion_vae_b200 import synth

pytestmark = pytest.mark.gpu

SELFTEST_BIT = 0x10


def test_bounded_wait_times_out_and_reports():
    B.device_error(reset=True)
    t0 = time.perf_counter()
    B.selftest_wait_timeout(20000)          # 20 ms
    code = B.device_error(reset=True)        # synchronises
    dt = time.perf_counter() - t0
    assert code == SELFTEST_BIT
    assert 0.015 <= dt < 5.0                 # waited about its limit, then returned
    assert B.device_error() == 0             # cleared


def test_context_usable_after_timeout():
    B.selftest_wait_timeout(5000)
    assert B.device_error(reset=True) == SELFTEST_BIT
    x, w, b = synth.conv_input(cin=64, cout=64, T=2, H=16, W=16, seed=0)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    y = B.causal_conv3d(to_cl(x), pk)
    assert_close(from_cl(y), O.causal_conv3d(x, w, b), torch.bfloat16, "after timeout")
    assert B.device_error() == 0
