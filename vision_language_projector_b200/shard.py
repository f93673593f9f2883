"""Partition one batch across ranks by sequence (host logic, no device work), and the
one exchange that data-parallel training of the projector has.

Images are independent units and every image's placeholder run lies inside one
sequence, so a batch splits into contiguous blocks of sequences with no exchange:
rank r projects the images whose runs lie in its sequences into its slice of the
embedding buffer. ``plan_shard`` returns the slices of every input a rank needs.

Training the projector on such shards, each rank's ``Projector.backward`` gives the
gradients of its sequences' share of the loss; the batch gradient of every parameter
is their sum over ranks (the loss is a sum over rows). ``allreduce_gradients`` adds
them in place across the process group (NCCL on GPUs) in one flat buffer.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import numpy as np


@dataclasses.dataclass(frozen=True)
class Shard:
    rank: int
    seq: slice          # sequences [start, stop)
    ids: slice          # flattened ids / embedding rows
    images: slice       # images [start, stop)
    views: slice        # views [start, stop) (grid_hw rows)
    patches: slice      # feature rows [start, stop)


def sequence_block(n_seq: int, world: int, rank: int) -> slice:
    """Contiguous, balanced block of sequences for `rank` (sizes differ by at most 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    base, extra = divmod(n_seq, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def plan_shard(image_seq: Sequence[int], views_per_image: Sequence[int], grid_hw: np.ndarray, n_seq: int,
               seq_len: int, world: int, rank: int) -> Shard:
    """`image_seq[i]` is the sequence holding image i's run (non-decreasing: images are
    ordered by sequence); `views_per_image[i]` its view count; `grid_hw` (n_views, 2)."""
    image_seq = np.asarray(image_seq, np.int64)
    if len(image_seq) and np.any(np.diff(image_seq) < 0):
        raise ValueError("images must be ordered by sequence")
    s = sequence_block(n_seq, world, rank)
    i0 = int(np.searchsorted(image_seq, s.start, side="left"))
    i1 = int(np.searchsorted(image_seq, s.stop, side="left"))
    vcum = np.concatenate([[0], np.cumsum(np.asarray(views_per_image, np.int64))])
    v0, v1 = int(vcum[i0]), int(vcum[i1])
    grid_hw = np.asarray(grid_hw, np.int64).reshape(-1, 2)
    pcum = np.concatenate([[0], np.cumsum(grid_hw[:, 0] * grid_hw[:, 1])])
    return Shard(rank, s, slice(s.start * seq_len, s.stop * seq_len), slice(i0, i1), slice(v0, v1),
                 slice(int(pcum[v0]), int(pcum[v1])))


def allreduce_gradients(grads: dict, group=None) -> None:
    """Sum every parameter gradient of ``grads`` over the ranks of ``group`` in place.

    Values may be tensors or lists of tensors (the middle layers' "W_mid" / "b_mid"),
    all of one dtype and device; keys are visited in sorted order on every rank. The
    tensors are packed into one buffer, so the exchange is a single all-reduce.

    The "features" entry (the gradient with respect to this rank's own feature rows)
    is left as it is: it belongs to the rank's shard of the batch, its size differs
    from rank to rank, and summing it across ranks would mix different patches. So
    ``Projector.backward``'s whole ``grads`` dict can be passed unchanged."""
    import torch
    import torch.distributed as dist

    tensors = []
    for key in sorted(grads):
        if key == "features":
            continue
        v = grads[key]
        tensors.extend(v if isinstance(v, (list, tuple)) else [v])
    if not tensors:
        return
    flat = torch.cat([t.reshape(-1) for t in tensors])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    offset = 0
    for t in tensors:
        n = t.numel()
        t.copy_(flat[offset:offset + n].view_as(t))
        offset += n
