"""Helpers shared by the GPU parity tests: layout conversion and the tolerances.

Tolerances (bf16 path): relative L2 error <= 1e-2 and max |error| <= 5e-2 * std
of the reference, over all compared elements; fp32 path: relative L2 <= 1e-4.
"""
import numpy as np
import torch

REL_L2_BF16 = 1e-2
MAX_ABS_BF16 = 5e-2
REL_L2_F32 = 1e-4


def to_cl(x, dtype=torch.bfloat16, device="cuda"):
    """Logical [C, T, H, W] (CPU tensor or array) -> channels-last [T, H, W, C] on device."""
    t = torch.as_tensor(np.asarray(x) if not isinstance(x, torch.Tensor) else x)
    return t.permute(1, 2, 3, 0).contiguous().to(device=device, dtype=dtype)


def from_cl(y):
    """Channels-last [T, H, W, C] device tensor -> float64 numpy [C, T, H, W]."""
    return y.detach().float().cpu().permute(3, 0, 1, 2).double().numpy()


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    rel = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)
    std = ref.std()
    mx = np.abs(d).max() / max(std, 1e-300)
    return rel, mx


def assert_close(got, ref, dtype, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rel, mx = errors(got, ref)
    if dtype == torch.float32:
        assert rel <= REL_L2_F32, f"{what}: rel L2 {rel:.3e} > {REL_L2_F32}"
    else:
        assert rel <= REL_L2_BF16, f"{what}: rel L2 {rel:.3e} > {REL_L2_BF16}"
        assert mx <= MAX_ABS_BF16, f"{what}: max abs / std {mx:.3e} > {MAX_ABS_BF16}"
    return rel, mx


def sample_voxels(T, H, W, n, seed=0, include_corners=True):
    """n voxel coordinates (t, h, w), always including the corners and edges."""
    rng = np.random.default_rng(seed)
    pts = set()
    if include_corners:
        for t in {0, T - 1}:
            for h in {0, H - 1}:
                for w in {0, W - 1}:
                    pts.add((t, h, w))
        pts.add((T - 1, H // 2, W - 1))
        pts.add((0, H - 1, W // 2))
    while len(pts) < n:
        pts.add((int(rng.integers(T)), int(rng.integers(H)), int(rng.integers(W))))
    return sorted(pts)
