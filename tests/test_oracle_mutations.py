"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each.

A pin set that passes a wrong oracle proves nothing; each mutation below is a
mistake a reader could make from the block's definition, and at least one pin
must fail on it.
"""
import math
import types

import numpy as np
import pytest

from oracle import oracle as O
from tests import oracle_pins as P
from video_diffusion_vae_b200 import synth


def _ns(**over):
    d = {k: getattr(O, k) for k in ("silu", "norm_silu", "causal_conv3d", "causal_conv3d_at",
                                    "upsample_nearest2x", "pixel_shuffle2x2", "resblock",
                                    "temporal_upsample2x")}
    d.update(over)
    return types.SimpleNamespace(**d)


def conv_flipped_time(x, wt, bias=None, cache=None, threads=None):
    return O.causal_conv3d(x, np.ascontiguousarray(np.asarray(wt)[:, :, ::-1]), bias, cache, threads)


def conv_centered_time(x, wt, bias=None, cache=None, threads=None):
    # pads one frame on each side instead of two in front
    x = np.asarray(x)
    xp = np.concatenate([x[:, 1:], np.zeros_like(x[:, :1])], axis=1)
    return O.causal_conv3d(xp, wt, bias, cache, threads)


def conv_no_bias(x, wt, bias=None, cache=None, threads=None):
    return O.causal_conv3d(x, wt, None, cache, threads)


def conv_transposed_spatial(x, wt, bias=None, cache=None, threads=None):
    return O.causal_conv3d(x, np.ascontiguousarray(np.swapaxes(np.asarray(wt), 3, 4)), bias, cache, threads)


def norm_variance_eps(x, gamma, beta, eps=1e-12, apply_silu=True):
    x = np.asarray(x, dtype=np.float64)
    C = x.shape[0]
    s = x / np.sqrt((x ** 2).mean(0, keepdims=True) + eps)
    s = s * np.asarray(gamma).reshape((C,) + (1,) * (x.ndim - 1)) + np.asarray(beta).reshape((C,) + (1,) * (x.ndim - 1))
    return s / (1 + np.exp(-s)) if apply_silu else s


def norm_no_root_c(x, gamma, beta, eps=1e-12, apply_silu=True):
    C = np.asarray(x).shape[0]
    g = np.asarray(gamma, dtype=np.float64) / math.sqrt(C)
    b = np.asarray(beta, dtype=np.float64)
    return O.norm_silu(x, g, b, eps, apply_silu)


def norm_sigmoid(x, gamma, beta, eps=1e-12, apply_silu=True):
    s = O.norm_silu(x, gamma, beta, eps, False)
    return 1 / (1 + np.exp(-s)) if apply_silu else s


def silu_wrong(s):
    return s / (1 + math.exp(s))


def shuffle_swapped(x):
    x = np.asarray(x)
    C4 = x.shape[0]
    idx = [4 * (k // 4) + 2 * (k % 2) + (k % 4) // 2 for k in range(C4)]
    return O.pixel_shuffle2x2(x[idx])


def upsample_bilinearish(x):
    y = O.upsample_nearest2x(x)
    y[:, :, 1::2] = 0.5 * (y[:, :, 1::2] + np.roll(y[:, :, 1::2], -1, axis=2))
    return y


def resblock_no_residual(x, p, threads=None):
    return O.resblock(x, p, threads) - np.asarray(x, dtype=np.float64)


def resblock_shortcut_on_normed(x, p, threads=None):
    if p.get("ws") is None:
        return O.resblock(x, p, threads)
    a = O.norm_silu(x, p["gamma1"], p["beta1"])
    h = O.causal_conv3d(O.norm_silu(O.causal_conv3d(a, p["w1"], p["b1"]), p["gamma2"], p["beta2"]),
                        p["w2"], p["b2"])
    return h + O.causal_conv3d(a, p["ws"], p["bs"])


MUTANTS = {
    "conv_flipped_time": _ns(causal_conv3d=conv_flipped_time),
    "conv_centered_time": _ns(causal_conv3d=conv_centered_time),
    "conv_no_bias": _ns(causal_conv3d=conv_no_bias),
    "conv_transposed_spatial": _ns(causal_conv3d=conv_transposed_spatial),
    "norm_variance_eps": _ns(norm_silu=norm_variance_eps),
    "norm_no_root_c": _ns(norm_silu=norm_no_root_c),
    "norm_sigmoid": _ns(norm_silu=norm_sigmoid),
    "silu_wrong": _ns(silu=silu_wrong),
    "shuffle_swapped": _ns(pixel_shuffle2x2=shuffle_swapped),
    "upsample_blend": _ns(upsample_nearest2x=upsample_bilinearish),
    "resblock_no_residual": _ns(resblock=resblock_no_residual),
}


def _fails(ns, extra=()):
    for check in list(P.ALL_CHECKS) + list(extra):
        try:
            check(ns)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    assert _fails(MUTANTS[name]), f"no pin failed for planted mistake {name}"


def test_pins_catch_shortcut_on_normalised_input():
    ns = _ns(resblock=resblock_shortcut_on_normed)
    assert _fails(ns, extra=[lambda o: P.check_resblock_library(o, synth)])


def test_real_oracle_passes_everything():
    assert not _fails(O, extra=[lambda o: P.check_resblock_library(o, synth),
                                lambda o: P.check_trunk_library(o, synth)])


# ------------------------------------------------- the causal cache
def conv_cache_reversed(x, wt, bias=None, cache=None, threads=None):
    # the cached frames taken newest first
    c = None if cache is None else np.ascontiguousarray(np.asarray(cache)[:, ::-1])
    return O.causal_conv3d(x, wt, bias, c, threads)


def conv_cache_ignored(x, wt, bias=None, cache=None, threads=None):
    return O.causal_conv3d(x, wt, bias, None, threads)


@pytest.mark.parametrize("mutant", [conv_cache_reversed, conv_cache_ignored])
def test_pins_catch_cache_mutant(mutant):
    assert _fails(_ns(causal_conv3d=mutant))


# ------------------------------------------------- the trunk's composition
def trunk_built(z, params, conv_before_upsample=False, head_norm=True,
                shuffle=O.pixel_shuffle2x2, drop_last_block=False):
    """The trunk from the oracle's layers, with one composition mistake planted
    on request (all False / default: the trunk as the oracle defines it)."""
    h = O.causal_conv3d(z, *params["conv_in"])
    stages = params["stages"]
    for s, st in enumerate(stages):
        blocks = st["blocks"][:-1] if drop_last_block and s == len(stages) - 1 else st["blocks"]
        for bp in blocks:
            h = O.resblock(h, bp)
        if st["up"] is not None:
            w, b = st["up"]
            h = O.upsample_nearest2x(O.causal_conv3d(h, w, b)) if conv_before_upsample \
                else O.causal_conv3d(O.upsample_nearest2x(h), w, b)
    hp = params["head"]
    if head_norm:
        a = O.norm_silu(h, hp["gamma"], hp["beta"])
    else:
        s_ = np.asarray(h) * np.asarray(hp["gamma"]).reshape(-1, 1, 1, 1) + \
            np.asarray(hp["beta"]).reshape(-1, 1, 1, 1)
        a = s_ / (1 + np.exp(-s_))
    return shuffle(O.causal_conv3d(a, hp["w"], hp["b"]))


TRUNK_MUTANTS = {
    "conv_before_upsample": dict(conv_before_upsample=True),
    "head_without_norm": dict(head_norm=False),
    "head_shuffle_swapped": dict(shuffle=shuffle_swapped),
    "last_block_dropped": dict(drop_last_block=True),
}


def _trunk_fails(**mistake):
    ns = types.SimpleNamespace(trunk=lambda z, params, threads=None: trunk_built(z, params, **mistake))
    try:
        P.check_trunk_library(ns, synth)
    except AssertionError:
        return True
    return False


def test_trunk_rebuild_without_mistake_passes():
    assert not _trunk_fails()


@pytest.mark.parametrize("name", sorted(TRUNK_MUTANTS))
def test_pins_catch_trunk_mutant(name):
    assert _trunk_fails(**TRUNK_MUTANTS[name]), f"the trunk pin passed planted mistake {name}"


# ------------------------------------------------- the temporal upsample
def temporal_first_doubled(x, first_chunk=True):
    return O.temporal_upsample2x(x, first_chunk=False)


def temporal_last_once(x, first_chunk=True):
    # keeps the last frame once instead of the first
    y = O.temporal_upsample2x(x, first_chunk=False)
    return y[:, :-1]


def temporal_blocked(x, first_chunk=True):
    # all copies of the first half, then all of the second: a tiled repeat
    y = O.temporal_upsample2x(x, first_chunk)
    return np.concatenate([y[:, 0::2], y[:, 1::2]], axis=1)


@pytest.mark.parametrize("mutant", [temporal_first_doubled, temporal_last_once, temporal_blocked])
def test_pins_catch_temporal_mutant(mutant):
    assert _fails(_ns(temporal_upsample2x=mutant))


def test_trunk_temporal_pin_catches_placement_and_count():
    """The library-built trunk pins the composition: the temporal step after
    the last upsample conv instead of the first, or a single step, fails."""
    def trunk_wrong(z, params, threads=None, temporal=False, first_chunk=True, stages=(1, 2)):
        h = O.causal_conv3d(z, *params["conv_in"])
        for s, st in enumerate(params["stages"]):
            for bp in st["blocks"]:
                h = O.resblock(h, bp)
            if st["up"] is not None:
                h = O.upsample_conv(h, *st["up"])
                if temporal and s in stages:
                    h = O.temporal_upsample2x(h, first_chunk)
        hp = params["head"]
        return O.head(h, hp["gamma"], hp["beta"], hp["w"], hp["b"])
    for stages in [(1, 2), (0,)]:
        ns = types.SimpleNamespace(trunk=lambda z, p, threads=None, temporal=False, first_chunk=True,
                                   st=stages: trunk_wrong(z, p, threads, temporal, first_chunk, st))
        with pytest.raises(AssertionError):
            P.check_trunk_temporal_library(ns, synth)
