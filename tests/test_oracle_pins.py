"""The CPU oracle against its pins (no GPU): closed forms, library special cases,
brute force and invariants.  See tests/oracle_pins.py for each check."""
import pytest

from oracle import oracle as O
from tests import oracle_pins as P
from video_diffusion_vae_b200 import synth


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(O)


def test_resblock_against_library():
    P.check_resblock_library(O, synth)


def test_trunk_against_library():
    P.check_trunk_library(O, synth)


def test_trunk_temporal_frames_and_causality():
    P.check_temporal_trunk_frames(O, synth)


def test_trunk_temporal_against_library():
    P.check_trunk_temporal_library(O, synth)
