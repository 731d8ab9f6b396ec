"""The row-slab split (video_diffusion_vae_b200/shard.py) on the CPU: gloo
ranks decode their rows of one video through the oracle's layers, exchanging
one halo row before every 3x3 conv; each rank's video rows equal the same
rows of the whole oracle decode, bit for bit, and rank 0 gathers the whole
video."""
import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.ports import free_port
from video_diffusion_vae_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_partition():
    for H, world in [(44, 1), (44, 2), (44, 3), (44, 8), (5, 3), (7, 7)]:
        parts = shard.partition(H, world)
        assert parts[0][0] == 0 and parts[-1][1] == H
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
        sizes = [r1 - r0 for r0, r1 in parts]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    assert shard.rows_at((11, 22), 16) == (176, 352)
    with pytest.raises(ValueError):
        shard.partition(3, 4)


def test_single_rank_halo_is_the_frame_padding():
    """One rank: both halo rows are the frame's zero padding (no process group
    needed); channels-last layout, rows on dim 1."""
    x = torch.randn(2, 3, 5, 8)                       # [T, rows, W, C]
    ext = shard.with_halo(x, 1)
    ext[:, 0] = 7.0
    ext[:, -1] = 7.0
    shard.exchange_halo(ext, 0, 1, 1)
    assert ext.shape == (2, 5, 5, 8)
    assert torch.equal(ext[:, 1:-1], x)
    assert not ext[:, 0].any() and not ext[:, -1].any()
    with pytest.raises(ValueError):
        shard.exchange_halo(torch.zeros(2, 2, 5, 8), 0, 1, 1)


# ---------------------------------------------------------------- gloo ranks
def _conv_rows(O, a, w, b, rank, world):
    """A 3x3 conv of this rank's rows: the input gets its halo, the conv runs
    over rows + 2 and the own rows are kept."""
    ext = shard.with_halo(torch.from_numpy(np.ascontiguousarray(a)), 2)
    shard.exchange_halo(ext, rank, world, 2)
    return O.causal_conv3d(ext.numpy(), w, b)[:, :, 1:-1]


def _upconv_rows(O, x, w, b, rank, world):
    ext = shard.with_halo(torch.from_numpy(np.ascontiguousarray(x)), 2)
    shard.exchange_halo(ext, rank, world, 2)
    return O.causal_conv3d(O.upsample_nearest2x(ext.numpy()), w, b)[:, :, 2:-2]


def _trunk_rows(O, z, params, rank, world, norm_after_exchange=False):
    def act(h, g, b):
        return O.norm_silu(h, g, b)

    def conv_act(h, g, b, w, bias):
        if norm_after_exchange:
            # a planted mistake: exchange the raw tensor and normalise the halo
            # too, so the frame's zero padding turns into SiLU(beta)
            ext = shard.with_halo(torch.from_numpy(np.ascontiguousarray(h)), 2)
            shard.exchange_halo(ext, rank, world, 2)
            return O.causal_conv3d(act(ext.numpy(), g, b), w, bias)[:, :, 1:-1]
        return _conv_rows(O, act(h, g, b), w, bias, rank, world)

    h = _conv_rows(O, z, *params["conv_in"], rank, world)
    for st in params["stages"]:
        for p in st["blocks"]:
            h1 = conv_act(h, p["gamma1"], p["beta1"], p["w1"], p["b1"])
            h2 = conv_act(h1, p["gamma2"], p["beta2"], p["w2"], p["b2"])
            skip = O.causal_conv3d(h, p["ws"], p["bs"]) if p.get("ws") is not None else h
            h = h2 + skip
        if st["up"] is not None:
            h = _upconv_rows(O, h, *st["up"], rank, world)
    hp = params["head"]
    return O.pixel_shuffle2x2(conv_act(h, hp["gamma"], hp["beta"], hp["w"], hp["b"]))


def _rank(rank, world, port, H, q, norm_after_exchange):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    from video_diffusion_vae_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        z, params = synth.trunk_input(T=2, H=H, W=4, widths=(16, 16, 8, 8), zc=6, seed=7)
        r0, r1 = shard.partition(H, world)[rank]
        zs = np.asarray(z.double().numpy())[:, :, r0:r1]
        mine = _trunk_rows(O, zs, params, rank, world, norm_after_exchange)
        whole = O.trunk(z, params)
        v0, v1 = shard.rows_at((r0, r1), 16)
        ok = mine.shape == whole[:, :, v0:v1].shape and np.array_equal(mine, whole[:, :, v0:v1])
        video = shard.gather_rows(torch.from_numpy(np.ascontiguousarray(mine)),
                                  shard.partition(H, world), 16, rank, world, 2)
        if rank == 0:
            ok = ok and np.array_equal(video.numpy(), whole)
        else:
            ok = ok and video is None
        q.put((rank, ok))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(world, port, H, norm_after_exchange=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank, args=(r, world, port, H, q, norm_after_exchange))
          for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(240)
    for p in ps:          # a rank stuck past the limit is ended, then reported
        if p.is_alive():
            p.terminate()
            p.join(10)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    return dict(q.get(timeout=10) for _ in range(world))


@pytest.mark.parametrize("world", [2, 3])
def test_row_split_trunk_equals_whole(world):
    got = _run(world, free_port(), H=5)
    assert all(got.values()), got


def test_row_split_needs_the_activated_halo():
    """Exchanging the raw tensor and normalising the halo rows as well gives
    the wrong border (SiLU(beta) where the frame pads with zeros)."""
    got = _run(2, free_port(), H=4, norm_after_exchange=True)
    assert not all(got.values())


# ------------------------------------------------- a subgroup of the ranks
def _sub_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sub = dist.new_group([1, 2])              # every rank creates it
        if rank in (1, 2):
            r, n = dist.get_rank(sub), dist.get_world_size(sub)
            parts = shard.partition(6, n)
            r0, r1 = parts[r]
            full = torch.arange(6 * 4, dtype=torch.float32).view(1, 6, 4)   # [T, rows, W]
            ext = shard.with_halo(full[:, r0:r1].clone(), 1)
            shard.exchange_halo(ext, r, n, 1, group=sub)
            want_top = full[:, r0 - 1] if r0 > 0 else torch.zeros(1, 4)
            want_bot = full[:, r1] if r1 < 6 else torch.zeros(1, 4)
            ok = torch.equal(ext[:, 0], want_top) and torch.equal(ext[:, -1], want_bot)
            got = shard.gather_rows(full[:, r0:r1], parts, 1, r, n, 1, group=sub)
            ok = ok and (torch.equal(got, full) if r == 0 else got is None)
            q.put((rank, ok))
        else:
            q.put((rank, True))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_halo_and_gather_on_a_subgroup():
    """Ranks {1, 2} of 3 as their own group: group rank 0 is global rank 1, so
    peers must be addressed by their global ranks."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    ps = [ctx.Process(target=_sub_rank, args=(r, 3, port, q)) for r in range(3)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    for p in ps:
        if p.is_alive():
            p.terminate()
            p.join(10)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    got = dict(q.get(timeout=10) for _ in range(3))
    assert all(got.values()), got


# --------------------------------------------------- the device path's host side
def test_slab_latents_halo_rows():
    """A slab's latents: its rows with the neighbouring rows above and below,
    zeros outside the frame."""
    z = torch.arange(2 * 3 * 5 * 4, dtype=torch.float32).view(1, 2, 3, 5, 4)
    top = shard.slab_latents(z, (0, 2))
    assert top.shape == (1, 2, 3, 4, 4)
    assert not top[:, :, :, 0].any() and torch.equal(top[:, :, :, 1:], z[:, :, :, 0:3])
    mid = shard.slab_latents(z, (2, 4))
    assert torch.equal(mid, z[:, :, :, 1:5])
    bot = shard.slab_latents(z, (4, 5))
    assert torch.equal(bot[:, :, :, :2], z[:, :, :, 3:5]) and not bot[:, :, :, 2].any()


def test_row_slab_halo_plan():
    """The library's plan for a slab (host only): the latents' re-layout and
    conv_in need no exchange; every other launch's input has the stage's own
    rows plus two, and the four stages' heights and widths follow the
    upsampling."""
    import ctypes
    from video_diffusion_vae_b200 import binding as B
    lib = B.load()
    w = (ctypes.c_int * 4)(512, 512, 256, 128)
    assert lib.wvae_decode_rows_steps() == lib.wvae_decode_trunk_launches() == 22
    plan = []
    for i in range(22):
        off, dims = ctypes.c_size_t(0), (ctypes.c_int * 4)()
        assert lib.wvae_decode_rows_halo(i, 4, 11, 78, w, ctypes.byref(off), dims) == 0
        plan.append((off.value, tuple(dims)))
    assert plan[0][1] == plan[1][1] == (0, 0, 0, 0)
    stage = {2: 0, 7: 1, 12: 2, 17: 3}
    for i in range(2, 22):
        s = max(k for k in stage if k <= i)
        st = stage[s]
        assert plan[i][1] == (4, (11 << st) + 2, 78 << st, (512, 512, 256, 128)[st]), (i, plan[i])
    ws = lib.wvae_decode_rows_workspace_bytes(4, 11, 78, w)
    assert all(off + 2 * d[0] * d[1] * d[2] * d[3] <= ws for off, d in plan)
    off, dims = ctypes.c_size_t(0), (ctypes.c_int * 4)()
    assert lib.wvae_decode_rows_halo(22, 4, 11, 78, w, ctypes.byref(off), dims) == 1


# ----------------------------------- the device driver's order, with gloo
class _FakeSlab:
    """Stands in for the library's row slab on the CPU: two launches that read
    a halo (steps 1 and 2) and one that does not (step 0).  Each launch checks
    that the halo rows of its input hold the neighbours' edge rows (or zeros
    at the frame's edges) and then writes its own rows from them, so a missed
    or misordered exchange changes the video."""

    def __init__(self, T, rows, W, r0, H):
        self.steps = 3
        self.rows, self.r0, self.H = rows, r0, H
        self.t = torch.zeros(T, rows + 2, W, 8, dtype=torch.bfloat16)
        self.halo = [None, self.t, self.t]
        self.ok = True

    def step(self, i, z_rows, video_rows):
        own = torch.arange(self.r0, self.r0 + self.rows, dtype=torch.float32)
        if i == 0:      # the slab's own rows hold their global row index + 1
            self.t[:, 1:-1] = (own + 1).view(1, -1, 1, 1).to(torch.bfloat16)
            return
        top = float(self.t[0, 0, 0, 0]); bot = float(self.t[0, -1, 0, 0])
        self.ok &= top == (self.r0 if self.r0 > 0 else 0.0)
        self.ok &= bot == (self.r0 + self.rows + 1 if self.r0 + self.rows < self.H else 0.0)
        if i == 2:      # video rows: the row's value + its neighbours', 16 video rows a latent row
            v = (self.t[:, :-2] + self.t[:, 1:-1] + self.t[:, 2:]).float()[..., 0]
            video_rows[0, :, :, :, :] = v.repeat_interleave(16, 1)[:, :, :1].unsqueeze(0)


def _driver_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T, H, W = 2, 5, 3
        parts = shard.partition(H, world)
        r0, r1 = parts[rank]
        fake = _FakeSlab(T, r1 - r0, W, r0, H)
        dec = shard.RowSplitDecoder(None, T, H, W, rank, world, device="cpu", slab=fake)
        z = torch.zeros(1, 48, T, H, W, dtype=torch.bfloat16)
        video = dec.decode(z)
        ok = fake.ok
        if rank == 0:
            rows = torch.arange(1, H + 1, dtype=torch.float32)
            pad = torch.cat([torch.zeros(1), rows, torch.zeros(1)])
            want = (pad[:-2] + pad[1:-1] + pad[2:]).repeat_interleave(16)
            ok = ok and video.shape == (1, 3, T, 16 * H, 16 * W) and \
                torch.equal(video[0, 0, 0, :, 0].float(), want)
        q.put((rank, bool(ok)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_split_driver_exchanges_and_gathers(world):
    """shard.RowSplitDecoder with gloo ranks: before every launch that reads
    a halo, the halo rows hold the neighbours' edge rows (zeros at the
    frame's edges); rank 0 receives every rank's video rows."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    ps = [ctx.Process(target=_driver_rank, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    for p in ps:
        if p.is_alive():
            p.terminate()
            p.join(10)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    got = dict(q.get(timeout=10) for _ in range(world))
    assert all(got.values()), got
