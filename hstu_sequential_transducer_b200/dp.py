"""Data-parallel plumbing for HSTU training over NCCL (one process per GPU).

Sequences are independent problems ("Ragged kernels": computation follows
each sequence's real length), so a batch shards across GPUs with no exchange
in the forward or the backward; the only collective of a training step is the
sum of the parameter gradients.

* ``lpt_shards`` splits ONE batch's sequences across ranks, balanced by the
  attention cost n^2 of each sequence (longest-processing-time-first: each
  sequence, largest first, goes to the rank with the smallest total so far).
  The most loaded rank then exceeds the least loaded one by at most one
  sequence's cost.
* ``BucketedAllReduce`` all-reduces each layer's gradients as soon as that
  layer's backward has been issued: the collective runs on the process
  group's own stream (NCCL) and overlaps the backward of the layers below;
  ``wait`` joins them before the gradients are read.

Both take plain tensors and a process group, so the same code runs over gloo
on CPU in the tests.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np
import torch


def sequence_costs(lengths: Sequence[int]) -> np.ndarray:
    """Attention cost of each sequence, n^2 (exact integers)."""
    n = np.asarray(lengths, dtype=np.int64)
    return n * n


def lpt_shards(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Indices of the sequences each of `world` ranks takes, balanced by n^2.

    Largest cost first (ties: lower index first), each to the rank with the
    smallest load so far (ties: lower rank).  Each rank's list is returned in
    increasing index order, so a shard keeps the batch's sequence order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = sequence_costs(lengths)
    order = sorted(range(len(cost)), key=lambda b: (-int(cost[b]), b))
    load = [0] * world
    shards: List[List[int]] = [[] for _ in range(world)]
    for b in order:
        r = min(range(world), key=lambda k: (load[k], k))
        shards[r].append(b)
        load[r] += int(cost[b])
    return [sorted(s) for s in shards]


def shard_loads(lengths: Sequence[int], shards: Sequence[Sequence[int]]) -> List[int]:
    cost = sequence_costs(lengths)
    return [int(sum(int(cost[b]) for b in s)) for s in shards]


class BucketedAllReduce:
    """Sum of per-layer gradient buckets over a process group, one
    asynchronous all-reduce per layer, issued as the layer's backward is."""

    def __init__(self, buckets: Sequence[torch.Tensor], dist, group=None):
        self.buckets = list(buckets)
        self.dist = dist
        self.group = group
        self.pending = []

    def layer_done(self, i: int):
        """Layer i's gradients are final in stream order: start their sum."""
        self.pending.append(self.dist.all_reduce(self.buckets[i], group=self.group,
                                                 async_op=True))

    def wait(self):
        """Orders the current stream after every started all-reduce."""
        for w in self.pending:
            w.wait()
        self.pending.clear()


def layer_buckets(flat: torch.Tensor, sizes: Sequence[int]) -> List[torch.Tensor]:
    """Contiguous views of `flat`, one of sizes[i] elements per layer."""
    out, o = [], 0
    for n in sizes:
        out.append(flat[o:o + n])
        o += n
    if o > flat.numel():
        raise ValueError("bucket sizes exceed the flat buffer")
    return out


def default_group_bucketing(step) -> Optional[BucketedAllReduce]:
    """Bucketed all-reduce of a TrainStep's gradients over the default process
    group, or None when running alone."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return None
    return BucketedAllReduce(layer_buckets(step.flat_grads, step.layer_grad_sizes), dist)
