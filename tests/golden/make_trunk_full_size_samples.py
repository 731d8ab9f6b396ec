"""Writes trunk_full_size_samples.txt: oracle values of the full-size decoder
trunk's video at a fixed set of pixels.

    python tests/golden/make_trunk_full_size_samples.py          (about 30 min on 8 cores)
    python tests/golden/make_trunk_full_size_samples.py --video  (about 80 min on 8 cores)

With --video it writes trunk_video_full_size_samples.txt instead: the same
latents decoded with the temporal 2x steps (oracle.trunk(temporal=True)),
video [1, 3, 13, 704, 1248]; the seam pixels are taken on frames 0, 1, 2, 5,
9 and 12.

The workload is the one the benchmark times: latents [1, 48, 4, 44, 78] drawn
by the seeded input module (seed 0), widths 512/512/256/128, video
[1, 3, 4, 704, 1248].  The whole video is computed by the fp64 CPU oracle
(oracle/oracle.py: conv_in, 4 stages of 2 residual blocks, 3 nearest-2x
upsample convs, norm_out + SiLU + head conv + 2x2 pixel shuffle).  This script
calls nothing but the oracle and the input generator; no value comes from the
CUDA library.

The file keeps, besides the sampled pixels, the whole video's standard
deviation and L2 norm, so that a test can apply the max-error bound relative to
the std over all output elements.

Pixels: every (channel, frame) at the crossings of a set of rows and columns
that lie on tile seams of the trunk's convs (a stage-3 tile of 16 x 16 voxels
covers 32 x 32 video pixels, stage 0's tiles 256 x 256) and on the frame's
edges, plus uniformly drawn pixels.
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

OUT = os.path.join(HERE, "trunk_full_size_samples.txt")
OUT_VIDEO = os.path.join(HERE, "trunk_video_full_size_samples.txt")
VIDEO_SEAM_FRAMES = (0, 1, 2, 5, 9, 12)
T, H, W = 4, 44, 78
SEED = 0
SEAM_ROWS = (0, 1, 15, 16, 31, 32, 63, 64, 255, 256, 351, 352, 511, 512, 687, 688, 702, 703)
SEAM_COLS = (0, 1, 31, 32, 255, 256, 447, 448, 511, 512, 623, 624, 1215, 1216, 1246, 1247)
N_RANDOM = 5000
PIXEL_SEED = 2024


def sample_pixels(C, Tn, Hn, Wn, seam_frames=None):
    frames = range(Tn) if seam_frames is None else seam_frames
    pts = set()
    for c in range(C):
        for t in frames:
            for h in SEAM_ROWS:
                for w in SEAM_COLS:
                    pts.add((c, t, h, w))
    rng = np.random.default_rng(PIXEL_SEED)
    while len(pts) < len(SEAM_ROWS) * len(SEAM_COLS) * C * len(frames) + N_RANDOM:
        pts.add((int(rng.integers(C)), int(rng.integers(Tn)), int(rng.integers(Hn)),
                 int(rng.integers(Wn))))
    return sorted(pts)


def main():
    from oracle import oracle as O
    from video_diffusion_vae_b200 import synth

    temporal = "--video" in sys.argv
    z, params = synth.trunk_input(T=T, H=H, W=W, seed=SEED)
    t0 = time.time()
    video = O.trunk(z, params, temporal=temporal)
    dt = time.time() - t0
    C, Tn, Hn, Wn = video.shape
    assert (C, Tn, Hn, Wn) == (3, 4 * T - 3 if temporal else T, 16 * H, 16 * W)
    pts = sample_pixels(C, Tn, Hn, Wn, VIDEO_SEAM_FRAMES if temporal else None)
    out = OUT_VIDEO if temporal else OUT
    with open(out, "w") as f:
        what = "with its temporal 2x steps (4T - 3 frames)" if temporal else "at full size"
        f.write(f"# Oracle (fp64) video of the decoder trunk {what}, sampled pixels.\n")
        f.write("# Written by tests/golden/make_trunk_full_size_samples.py (oracle + seeded inputs only).\n")
        f.write(f"# workload: latents [1,48,{T},{H},{W}] seed {SEED}, widths 512/512/256/128\n")
        f.write(f"# oracle seconds: {dt:.0f}\n")
        f.write(f"std {float(video.std())!r}\n")
        f.write(f"l2 {float(np.linalg.norm(video))!r}\n")
        f.write(f"count {len(pts)}\n")
        for (c, t, h, w) in pts:
            f.write(f"{c} {t} {h} {w} {float(video[c, t, h, w])!r}\n")
    print(f"wrote {len(pts)} samples to {out} ({dt:.0f} s of oracle)")


if __name__ == "__main__":
    main()
