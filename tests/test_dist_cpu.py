"""Data-parallel host logic of bench.py on CPU: two gloo ranks.

Sequences are independent ("Ragged kernels": each sequence is its own
problem), so the gradient of a batch is the sum of the gradients of its
sequences.  With weak scaling every rank takes its own sequences and one
all-reduce (sum) of the gradient buffer gives every rank the batch gradient;
the job's step time is the slowest rank's.  This runs the bench's own helpers
(`allreduce_grads`, `max_over_ranks`, `rank_data_seed`) and the package's
data-parallel pieces (`dp.lpt_shards`, `dp.BucketedAllReduce`) over gloo, with
the fp64 oracle standing in for the GPU step.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

LENGTHS = [5, 9, 3, 7]        # rank r takes sequences r, r + 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _workload():
    from hstu_sequential_transducer_b200 import workloads as W
    return W.custom(LENGTHS, d=16, H=2, N=16.0, dtype="f32", layers=2, seed=21, backward=True,
                    with_bias=True, with_affine=True)


def _oracle_grads(w):
    """Flat fp64 vector of every layer's parameter gradients (fixed order)."""
    from oracle import hstu_ref as R
    plist = [R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)
             for p in w.params]
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    _, _, grads = R.stack_forward_backward(w.x, w.seq_offsets, w.timestamps, w.num_targets,
                                           plist, cfg, w.dy)
    parts = []
    for g in grads:
        for name in ("dW1", "dW2", "db1", "db2", "dgamma", "dbeta", "drab_pos", "drab_time"):
            v = getattr(g, name)
            if v is not None:
                parts.append(np.asarray(v, np.float64).ravel())
    return np.concatenate(parts)


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from hstu_sequential_transducer_b200 import workloads as W
        w = _workload()
        mine = W.subset(w, list(range(rank, len(LENGTHS), world)))
        flat = torch.from_numpy(_oracle_grads(mine))
        bench.allreduce_grads(flat, dist)
        ms = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
        out[rank] = (flat.numpy().copy(), ms, bench.rank_data_seed(rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_allreduce_and_timing():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    whole = _oracle_grads(_workload())
    for r in range(world):
        flat, ms, seed = res[r]
        # the all-reduced shard gradients are the whole batch's gradient
        np.testing.assert_allclose(flat, whole, rtol=1e-12, atol=1e-12)
        assert ms == 11.0                       # the slowest rank's time
    assert res[0][2] != res[1][2]               # ranks draw different sequences


def _oracle_layer_grads(w):
    """Per layer, the flat fp64 vector of its parameter gradients."""
    from oracle import hstu_ref as R
    plist = [R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)
             for p in w.params]
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    _, _, grads = R.stack_forward_backward(w.x, w.seq_offsets, w.timestamps, w.num_targets,
                                           plist, cfg, w.dy)
    out = []
    for g in grads:
        parts = [np.asarray(getattr(g, n), np.float64).ravel()
                 for n in ("dW1", "dW2", "db1", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")
                 if getattr(g, n) is not None]
        out.append(np.concatenate(parts))
    return out


SPLIT_LENGTHS = [9, 3, 12, 5, 7, 2]


def _split_workload():
    from hstu_sequential_transducer_b200 import workloads as W
    return W.custom(SPLIT_LENGTHS, d=16, H=2, N=16.0, dtype="f32", layers=3, seed=23,
                    backward=True, with_bias=True, with_affine=True)


def _rank_split_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from hstu_sequential_transducer_b200 import dp
        w = _split_workload()
        mine = bench.split_shard(w, rank, world)
        per_layer = _oracle_layer_grads(mine)
        flat = torch.zeros(sum(len(g) for g in per_layer), dtype=torch.float64)
        buckets = dp.layer_buckets(flat, [len(g) for g in per_layer])
        bk = dp.BucketedAllReduce(buckets, dist)
        # the backward visits layers top-down; each layer's sum starts as soon
        # as its gradients are written, while the layers below still run
        for i in range(len(per_layer) - 1, -1, -1):
            buckets[i].copy_(torch.from_numpy(per_layer[i]))
            bk.layer_done(i)
        bk.wait()
        out[rank] = (flat.numpy().copy(), sorted(dp.lpt_shards(w.lengths, world)[rank]))
    finally:
        dist.destroy_process_group()


def test_two_rank_split_batch_bucketed_allreduce():
    """One batch split across 2 ranks by n^2 (LPT), per-layer buckets summed
    asynchronously in backward order: every rank ends with the whole batch's
    gradient, and the shards cover every sequence once."""
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_split_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    whole = np.concatenate(_oracle_layer_grads(_split_workload()))
    for r in range(world):
        np.testing.assert_allclose(res[r][0], whole, rtol=1e-12, atol=1e-12)
    cover = sorted(res[0][1] + res[1][1])
    assert cover == list(range(len(SPLIT_LENGTHS)))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_lpt_split_balance(world):
    """LPT on the training batch's lengths: a partition of the sequences whose
    heaviest and lightest shards differ by at most the largest n^2 (the last
    sequence placed on the heaviest shard went to the lightest one)."""
    from hstu_sequential_transducer_b200 import dp
    from hstu_sequential_transducer_b200 import workloads as W
    lengths = W.training().lengths
    shards = dp.lpt_shards(lengths, world)
    assert sorted(b for s in shards for b in s) == list(range(len(lengths)))
    loads = dp.shard_loads(lengths, shards)
    assert max(loads) - min(loads) <= int(np.max(lengths)) ** 2
    assert sum(loads) == int(np.sum(np.asarray(lengths, np.int64) ** 2))
    # Graham: LPT is within 4/3 of the optimum, which is at least the average load
    assert max(loads) <= (4 / 3) * sum(loads) / world + 1e-9 or world == 1


def test_lpt_split_small_cases():
    from hstu_sequential_transducer_b200 import dp
    assert dp.lpt_shards([3, 1, 2], 1) == [[0, 1, 2]]
    # costs 64, 49, 36, 25: 64 -> r0, 49 -> r1, 36 -> r1 (49 < 64), 25 -> r0
    assert dp.lpt_shards([8, 7, 6, 5], 2) == [[0, 3], [1, 2]]
    assert dp.lpt_shards([], 3) == [[], [], []]
    assert dp.lpt_shards([4], 3) == [[0], [], []]
    with pytest.raises(ValueError):
        dp.lpt_shards([1], 0)
