"""Row-slab split of one decode over ranks: the host side of a spatial split.

The FastVideo Wan2.2 VAE decoder spreads one decode over several GPUs of a
node - every rank calls it with the same latents, rank 0 receives the video
(README, "Use"), 3.57x faster at 4 GPUs ("Performance and memory") - without
saying how it splits the work.  This module holds the host side of a split
over frame rows:

* partition(): the latent rows each rank owns.  At stage s of the trunk a rank
  owns the rows [2^s r0, 2^s r1) of that stage's resolution and, in the video,
  the rows [16 r0, 16 r1).
* gather_rows(): rank 0 assembles the whole output from the ranks' rows
  (the pages' decoder returns the video on rank 0).
* exchange_halo(): the one-row halo every 3x3 conv needs (the causal 3x3x3
  convs, the upsample convs, the head).  A rank keeps each conv input with
  one extra row above and below its own rows; before the conv the extra rows
  are filled with the neighbours' edge rows, or with zeros at the frame's
  top and bottom.  The exchanged tensor is the conv's INPUT after norm and
  SiLU, since the frame's zero padding applies after the activation.
  Everything else on the path (norm, SiLU, residual, shortcut, pixel
  shuffle) is per voxel and needs no exchange.

With the extra rows in place a conv computed over rows + 2 rows gives its own
rows exactly (the two outer rows are discarded, or overwritten by the next
exchange), so the convs themselves need no change.  Works on CPU tensors
(gloo) and CUDA tensors (NCCL) alike.

On the device (decode_rows): the library's row-slab decode keeps every
tensor with one halo row per side and runs one launch at a time
(wvae_decode_rows_*); between launches the caller fills the halo rows of the
next conv's input.  The upsample convs write the next stage's slab (own rows
plus one halo row each side) directly, and the head writes the rank's own
video rows.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def partition(H: int, world: int) -> list[tuple[int, int]]:
    """Contiguous row ranges [r0, r1) of H rows over `world` ranks, sizes
    differing by at most one (the first H % world ranks take the extra row)."""
    if world < 1 or H < world:
        raise ValueError(f"cannot split {H} rows over {world} ranks")
    base, extra = divmod(H, world)
    out, r0 = [], 0
    for r in range(world):
        r1 = r0 + base + (1 if r < extra else 0)
        out.append((r0, r1))
        r0 = r1
    return out


def rows_at(part: tuple[int, int], scale: int) -> tuple[int, int]:
    """A rank's rows at a resolution `scale` times the latents'."""
    return part[0] * scale, part[1] * scale


def with_halo(x: torch.Tensor, row_dim: int) -> torch.Tensor:
    """A copy of x with one (zero) row added above and below along row_dim."""
    shape = list(x.shape)
    shape[row_dim] += 2
    out = x.new_zeros(shape)
    out.narrow(row_dim, 1, x.shape[row_dim]).copy_(x)
    return out


def _peer(group, r: int) -> int:
    """The global rank of rank r of `group` (torch addresses peers globally)."""
    return r if group is None else dist.get_global_rank(group, r)


def exchange_halo(x_ext: torch.Tensor, rank: int, world: int, row_dim: int, group=None) -> None:
    """Fill the halo rows of x_ext in place.

    x_ext holds, along row_dim, one halo row, the rank's own rows, one halo row.
    Row 0 receives the last own row of rank - 1 (zeros on rank 0); the last row
    receives the first own row of rank + 1 (zeros on the last rank).  `rank`
    and `world` are this process's rank in `group` and the group's size (the
    default group when None).  Every rank of the group must call it (ranks
    with one neighbour exchange with it alone)."""
    n = x_ext.shape[row_dim]
    if n < 3:
        raise ValueError("x_ext needs at least one own row between the two halo rows")
    first = x_ext.narrow(row_dim, 1, 1).contiguous()
    last = x_ext.narrow(row_dim, n - 2, 1).contiguous()
    top = torch.zeros_like(first)
    bottom = torch.zeros_like(first)
    ops = []
    if rank > 0:
        ops.append(dist.P2POp(dist.isend, first, _peer(group, rank - 1), group))
        ops.append(dist.P2POp(dist.irecv, top, _peer(group, rank - 1), group))
    if rank < world - 1:
        ops.append(dist.P2POp(dist.isend, last, _peer(group, rank + 1), group))
        ops.append(dist.P2POp(dist.irecv, bottom, _peer(group, rank + 1), group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    x_ext.narrow(row_dim, 0, 1).copy_(top)
    x_ext.narrow(row_dim, n - 1, 1).copy_(bottom)


def gather_rows(mine: torch.Tensor, parts: list[tuple[int, int]], scale: int, rank: int,
                world: int, row_dim: int, group=None):
    """Rank 0 of the group receives every rank's rows (`mine`: this rank's rows
    at `scale` times the latent resolution, along row_dim) and returns the
    whole tensor; the other ranks send theirs and return None.  Every rank of
    the group must call it.  Rank 0 sizes each receive buffer from its own
    tensor, so every rank's `mine` must have rank 0's dtype and rank 0's shape
    apart from row_dim (whose length must be the rank's row count: checked).
    `rank` and `world` are this process's rank in `group` and its size."""
    r0, r1 = rows_at(parts[rank], scale)
    if mine.shape[row_dim] != r1 - r0:
        raise ValueError(f"rank {rank} holds {mine.shape[row_dim]} rows, its part has {r1 - r0}")
    if rank != 0:
        dist.send(mine.contiguous(), _peer(group, 0), group)
        return None
    pieces = [mine.contiguous()]
    for src in range(1, world):
        a, b = rows_at(parts[src], scale)
        shape = list(mine.shape)
        shape[row_dim] = b - a
        buf = mine.new_empty(shape)
        dist.recv(buf, _peer(group, src), group)
        pieces.append(buf)
    return torch.cat(pieces, dim=row_dim)


# ------------------------------------------------------------ device decode
def slab_latents(z: torch.Tensor, part: tuple[int, int]) -> torch.Tensor:
    """The latents of a rank's rows with one halo row above and below, taken
    from the whole latents z [1, C, T, H, W] (zeros outside the frame)."""
    r0, r1 = part
    H = z.shape[3]
    out = z.new_zeros(z.shape[:3] + (r1 - r0 + 2,) + z.shape[4:])
    a, b = max(r0 - 1, 0), min(r1 + 1, H)
    out[:, :, :, a - (r0 - 1):b - (r0 - 1)] = z[:, :, :, a:b]
    return out.contiguous()


class RowSplitDecoder:
    """This rank's part of decodes split by latent rows over the ranks of
    `group`: its row slab (workspace and halo views), its latents with their
    halo rows and its video rows, set up once and reused by decode().
    `slab` may be given (any object with the RowSlab interface: steps, halo,
    step(i, z_rows, video_rows)); by default the library's row slab."""

    def __init__(self, trunk, T: int, H: int, W: int, rank: int, world: int, group=None,
                 device="cuda", slab=None):
        self.rank, self.world, self.group = rank, world, group
        self.parts = partition(H, world)
        r0, r1 = self.parts[rank]
        if slab is None:
            from video_diffusion_vae_b200 import binding as B
            slab = B.RowSlab(trunk, T, r1 - r0, W, device=device)
        self.slab = slab
        self.video = torch.empty((1, 3, T, 16 * (r1 - r0), 16 * W), dtype=torch.bfloat16,
                                 device=device)

    def decode(self, z, gather: bool = True):
        """z: the whole latents [1, 48, T, H, W] (every rank passes the same).
        Returns the whole video on rank 0 (gather=True; None elsewhere) or this
        rank's video rows."""
        zr = slab_latents(z, self.parts[self.rank])
        sl = self.slab
        for i in range(sl.steps):
            if sl.halo[i] is not None:
                exchange_halo(sl.halo[i], self.rank, self.world, 1, self.group)
            sl.step(i, zr, self.video)
        if not gather:
            return self.video
        return gather_rows(self.video, self.parts, 16, self.rank, self.world, 3, self.group)


def decode_rows(z, trunk, rank: int, world: int, group=None, gather: bool = True):
    """One decode split over the ranks of `group` by latent rows (every rank
    passes the same latents z [1, 48, T, H, W], bf16, on its GPU).  Each rank
    decodes its rows through the library's row-slab steps, exchanging the
    halo rows of every 3x3 conv's input with its neighbours (NCCL point-to-
    point for CUDA tensors).  Returns the whole video on rank 0 (gather=True,
    as the pages' decoder does) or this rank's video rows."""
    _, _, T, H, W = z.shape
    dec = RowSplitDecoder(trunk, T, H, W, rank, world, group, device=z.device)
    return dec.decode(z, gather)


def decode_rows_emulated(z, trunk, world: int):
    """The row split on one device: `world` slabs step in lockstep and the halo
    rows are copied between them (standing in for the NCCL exchange).
    Returns the assembled video."""
    from video_diffusion_vae_b200 import binding as B
    _, _, T, H, W = z.shape
    parts = partition(H, world)
    slabs = [B.RowSlab(trunk, T, r1 - r0, W, device=z.device) for r0, r1 in parts]
    zs = [slab_latents(z, p) for p in parts]
    videos = [torch.empty((1, 3, T, 16 * (r1 - r0), 16 * W), dtype=torch.bfloat16, device=z.device)
              for r0, r1 in parts]
    for i in range(slabs[0].steps):
        views = [sl.halo[i] for sl in slabs]
        if views[0] is not None:
            for r, v in enumerate(views):
                n = v.shape[1]
                if r > 0:
                    v[:, 0].copy_(views[r - 1][:, views[r - 1].shape[1] - 2])
                else:
                    v[:, 0].zero_()
                if r < world - 1:
                    v[:, n - 1].copy_(views[r + 1][:, 1])
                else:
                    v[:, n - 1].zero_()
        for sl, zr, vd in zip(slabs, zs, videos):
            sl.step(i, zr, vd)
    return torch.cat(videos, dim=3)
