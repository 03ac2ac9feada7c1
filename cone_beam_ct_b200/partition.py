"""One DRR job split over GPUs: detector rows (and with them views) divided
among ranks, the volume replicated on every rank (diffct page, "Multi-GPU
and multi-node": views partitioned across processes, each holding the whole
volume, launched with torchrun over NCCL).  One process per GPU with
torch.distributed; every step of the path runs in libdrr.so's kernels, and
the only exchanges are the collectives below:

* ``broadcast_volume`` -- the volume once from one rank to all (NCCL);
* the forward needs nothing more: every ray is independent;
* ``adjoint_partitioned`` -- each rank scatters its rays' gradient into its
  own gradient volume, then one all-reduce (sum) gives every rank the whole
  volume gradient.

A rank's share of a B x H x W image stack is a contiguous run of its B*H
detector rows, view-major, so shares differ by at most one row and any
number of ranks up to B*H works (a 4-view job splits over 8 GPUs).  The run
is rendered as whole views (one call) and at most two partial views; a
partial view is a block of rows [r0, r0 + h) rendered as an image of h rows
through intrinsics whose principal point row is moved by r0: with K' = T K,
T = [[1, 0, 0], [0, 1, -r0], [0, 0, 1]], row r of the block maps to the same
ray as detector row r0 + r (K'^-1 (u, r, 1) = K^-1 (u, r + r0, 1)), so K'
differs from K only in cy' = cy - r0 * K[2][2].
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np

from . import drr


@dataclasses.dataclass(frozen=True)
class Segment:
    """Views [view0, view0 + n_views), rows [row0, row0 + rows) of each, at
    element ``offset`` of the rank's local image buffer (row-major, W
    columns)."""
    view0: int
    n_views: int
    row0: int
    rows: int
    offset: int


def shard_rows(B: int, H: int, world: int, rank: int) -> Tuple[int, int]:
    """The rank's run [start, stop) of the B*H detector rows (view-major):
    balanced, contiguous, in rank order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    total = B * H
    return rank * total // world, (rank + 1) * total // world


def segments(B: int, H: int, W: int, start: int, stop: int) -> List[Segment]:
    """The run [start, stop) of flattened rows as at most three calls: a
    partial first view, whole views, a partial last view."""
    out: List[Segment] = []
    off = 0
    g = start
    while g < stop:
        view, row = divmod(g, H)
        if row == 0 and stop - g >= H:
            n = (stop - g) // H                   # whole views
            out.append(Segment(view, n, 0, H, off))
            g += n * H
            off += n * H * W
        else:
            rows = min(H - row, stop - g)        # a block of rows of one view
            out.append(Segment(view, 1, row, rows, off))
            g += rows
            off += rows * W
    return out


def row_block_K(K: Sequence[float], row0: int) -> np.ndarray:
    """Intrinsics of the block of detector rows starting at ``row0``: the
    principal point row moved by row0 (see the module docstring)."""
    k = np.asarray(K, dtype=np.float64).reshape(9).copy()
    k[5] = k[5] - row0 * k[8]
    return k.astype(np.float32)


def world_and_rank() -> Tuple[int, int]:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


class Partition:
    """This rank's share of a B x H x W image stack."""

    def __init__(self, B: int, H: int, W: int, world: Optional[int] = None,
                 rank: Optional[int] = None):
        if world is None or rank is None:
            world, rank = world_and_rank()
        self.B, self.H, self.W, self.world, self.rank = B, H, W, world, rank
        self.start, self.stop = shard_rows(B, H, world, rank)
        self.segments = segments(B, H, W, self.start, self.stop)

    @property
    def rows(self) -> int:
        """Detector rows of this rank (its image buffer holds rows * W floats)."""
        return self.stop - self.start

    @property
    def rays(self) -> int:
        return self.rows * self.W

    def local_slice(self) -> slice:
        """Where this rank's rows sit in the flattened B*H*W image stack."""
        return slice(self.start * self.W, self.stop * self.W)


def _pose_rows(Rt, seg: Segment):
    return Rt.reshape(-1, 12)[seg.view0:seg.view0 + seg.n_views]


def _seg_K(K, seg: Segment):
    return K if seg.row0 == 0 else row_block_K(K, seg.row0)


def _flat(t, seg: Segment, W: int):
    return t.reshape(-1)[seg.offset:seg.offset + seg.n_views * seg.rows * W]


def render_partitioned(part: Partition, vol, dtype, layout, dims, spacing, origin, K, Rt,
                       n_samples, density_factor, mode, out_local, stream=None,
                       render: Callable = None):
    """Forward of this rank's rows into ``out_local`` (part.rows * W floats;
    Rt: the device array of all B poses).  ``render`` defaults to
    drr.drr_render (same signature)."""
    render = drr.drr_render if render is None else render
    for seg in part.segments:
        render(vol, dtype, layout, dims, spacing, origin, _seg_K(K, seg), _pose_rows(Rt, seg),
               seg.n_views, seg.rows, part.W, n_samples, density_factor, mode,
               _flat(out_local, seg, part.W), stream=stream)


def adjoint_partitioned(part: Partition, dims, spacing, origin, K, Rt, n_samples,
                        density_factor, mode, grad_out_local, fwd_out_local, grad_vol,
                        workspace=None, stream=None, adjoint: Callable = None,
                        reduce: bool = True):
    """Volume gradient of this rank's rows accumulated into ``grad_vol`` (a
    workspace, when given, lets dense views take the record path), then,
    with ``reduce`` and a process group of more than one rank, one all-reduce
    (sum) over ranks, so every rank holds the gradient of the whole job.
    ``adjoint`` defaults to drr.drr_render_adjoint_ws with ``workspace``, or
    drr.drr_render_adjoint without one (same signatures)."""
    for seg in part.segments:
        fwd = None if fwd_out_local is None else _flat(fwd_out_local, seg, part.W)
        args = (dims, spacing, origin, _seg_K(K, seg), _pose_rows(Rt, seg), seg.n_views,
                seg.rows, part.W, n_samples, density_factor, mode,
                _flat(grad_out_local, seg, part.W), fwd, grad_vol)
        if adjoint is not None:
            adjoint(*args, stream=stream)
        elif workspace is not None:
            drr.drr_render_adjoint_ws(*args, workspace, stream=stream)
        else:
            drr.drr_render_adjoint(*args, stream=stream)
    if reduce:
        allreduce_sum(grad_vol)


def allreduce_sum(t) -> None:
    """Sum ``t`` over the ranks in place (no-op without a process group)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)


def broadcast_volume(vol, src: int = 0) -> None:
    """The volume from rank ``src`` to every rank, in place (no-op without a
    process group)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.broadcast(vol, src=src)
