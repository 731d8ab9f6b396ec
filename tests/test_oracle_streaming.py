"""The streaming decode's premise, pinned on the oracle alone: with every
causal conv reading its two front frames from the previous chunk (the cache),
decoding the latents chunk by chunk equals decoding them at once (causality).
The GPU's chunked decode is checked against its own whole decode in the GPU
tests; this shows the scheme itself is exact."""
import numpy as np
import pytest

from oracle import oracle as O
from video_diffusion_vae_b200 import synth


def _trunk_chunk(z, params, caches, first, temporal=False):
    """One chunk of the oracle trunk; caches[i] holds the last two input frames
    of causal conv i from the previous chunk and is replaced by this chunk's."""
    it = iter(range(18))

    def cconv(x, w, b):
        i = next(it)
        y = O.causal_conv3d(x, w, b, cache=None if first else caches[i])
        caches[i] = x[:, -2:].copy()
        return y

    h = cconv(z, *params["conv_in"])
    for s, st in enumerate(params["stages"]):
        for p in st["blocks"]:
            a1 = O.norm_silu(h, p["gamma1"], p["beta1"])
            h1 = cconv(a1, p["w1"], p["b1"])
            a2 = O.norm_silu(h1, p["gamma2"], p["beta2"])
            h = cconv(a2, p["w2"], p["b2"]) + h       # the trunk's blocks keep their width
        if st["up"] is not None:
            h = O.upsample_conv(h, *st["up"])        # per frame: no cache
            if temporal and s < 2:                   # the first two stages
                h = O.temporal_upsample2x(h, first_chunk=first)
    hp = params["head"]
    a = O.norm_silu(h, hp["gamma"], hp["beta"])
    return O.pixel_shuffle2x2(cconv(a, hp["w"], hp["b"]))


@pytest.mark.parametrize("chunks", [(2, 2), (2, 3)])
def test_oracle_chunked_trunk_equals_whole(chunks):
    T = sum(chunks)
    z, params = synth.trunk_input(T=T, H=2, W=2, widths=(64, 64, 64, 64), seed=7)
    whole = O.trunk(z, params)
    zn = z.double().numpy()
    caches, parts, t0 = [None] * 18, [], 0
    for i, n in enumerate(chunks):
        parts.append(_trunk_chunk(zn[:, t0:t0 + n], params, caches, first=(i == 0)))
        t0 += n
    np.testing.assert_allclose(np.concatenate(parts, axis=1), whole, rtol=0, atol=1e-12)


def test_oracle_chunk_without_cache_differs():
    """The pin can fail: dropping the cache (zero front frames in the second
    chunk) changes the second chunk's video."""
    z, params = synth.trunk_input(T=4, H=2, W=2, widths=(64, 64, 64, 64), seed=7)
    whole = O.trunk(z, params)
    zn = z.double().numpy()
    second = _trunk_chunk(zn[:, 2:], params, [None] * 18, first=True)
    assert np.abs(second - whole[:, 2:]).max() > 1e-3


@pytest.mark.parametrize("chunks", [(2, 2), (2, 3)])
def test_oracle_chunked_temporal_trunk_equals_whole(chunks):
    """With temporal upsampling: the first chunk keeps its first frame once,
    later chunks double every frame; chunk by chunk gives 4T - 3 frames equal
    to the whole decode's."""
    T = sum(chunks)
    z, params = synth.trunk_input(T=T, H=2, W=2, widths=(64, 64, 64, 64), seed=9)
    whole = O.trunk(z, params, temporal=True)
    assert whole.shape[1] == 4 * T - 3
    zn = z.double().numpy()
    caches, parts, t0 = [None] * 18, [], 0
    for i, n in enumerate(chunks):
        parts.append(_trunk_chunk(zn[:, t0:t0 + n], params, caches, first=(i == 0), temporal=True))
        t0 += n
    np.testing.assert_allclose(np.concatenate(parts, axis=1), whole, rtol=0, atol=1e-12)
