"""Row-sharded triangle update over the ranks of a torch.distributed process group.

"Big mode" for complexes whose pair tensor does not fit one GPU: rank g holds rows
[bounds[g], bounds[g+1]) of z and the mask (whole 128-row blocks) and produces the same rows
of the update (see include/trimul.h, tri_mul_shard_project / tri_mul_shard_finish):

  phase 1   a, b of the rank's rows                      (the CUDA library)
  exchange  every rank's b (and, incoming, every a)      (one all-gather each, torch.distributed)
  phase 2   contraction and output gate of the rank's rows (the CUDA library)

Outgoing (x_ij = sum_k a_ik b_jk) needs this rank's a rows and all of b; incoming
(x_ij = sum_k a_ki b_kj) needs a and b rows k from every rank. The exchange here is the
plain collective; the phase-2 entry point also accepts other GPUs' buffers directly (peer
mappings), which this module does not set up. Only host-side bookkeeping lives here.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .trimul import shard_bounds


def gather_rows(t: torch.Tensor, bounds: list, rank: int, group=None) -> list:
    """Every rank's [B, C, R_g, N] tensor (its rows of the planes), as a list indexed by rank.
    Shards of unequal size travel padded to the largest one."""
    world = len(bounds) - 1
    sizes = [bounds[g + 1] - bounds[g] for g in range(world)]
    rmax = max(sizes)
    if t.shape[2] != sizes[rank]:
        raise ValueError(f"rank {rank} holds {t.shape[2]} rows, its shard has {sizes[rank]}")
    send = t
    if sizes[rank] != rmax:
        send = torch.zeros((t.shape[0], t.shape[1], rmax, t.shape[3]), dtype=t.dtype, device=t.device)
        send[:, :, :sizes[rank]] = t
    bufs = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(bufs, send.contiguous(), group=group)
    return [bufs[g] if sizes[g] == rmax else bufs[g][:, :, :sizes[g]].contiguous() for g in range(world)]


class RowShardedTriMul:
    """One triangle update split by rows over the ranks of `group` (one GPU per rank).

    layer: the rank's TriMulLayer (same weights on every rank). project / finish replace the
    two phases (signatures of TriMulLayer.shard_project / shard_finish), e.g. for tests of the
    bookkeeping without a GPU.
    """

    def __init__(self, layer=None, group=None, project=None, finish=None):
        self.layer = layer
        self.group = group
        self._project = project or layer.shard_project
        self._finish = finish or layer.shard_finish

    def bounds(self, N: int) -> list:
        return shard_bounds(N, dist.get_world_size(self.group))

    def forward(self, z_rows: torch.Tensor, mask_rows, N: int, direction: str, out=None):
        rank = dist.get_rank(self.group)
        bounds = self.bounds(N)
        row0 = bounds[rank]
        if z_rows.shape[1] != bounds[rank + 1] - row0:
            raise ValueError(f"rank {rank} must hold rows [{row0}, {bounds[rank + 1]}) of z")
        a, b = self._project(z_rows, mask_rows, row0, N)
        b_all = gather_rows(b, bounds, rank, self.group)
        if direction == "incoming":
            a_all = gather_rows(a, bounds, rank, self.group)
        else:
            a_all = [None] * (len(bounds) - 1)
            a_all[rank] = a
        return self._finish(z_rows, mask_rows, row0, N, direction, bounds, a_all, b_all, out=out)

    __call__ = forward
