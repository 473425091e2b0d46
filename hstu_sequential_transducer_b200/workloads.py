"""Seeded synthetic workloads for the HSTU layer.

This module only draws random inputs (lengths, values, timestamps, weights);
it holds none of the layer's arithmetic.  The CUDA path and the fp64 oracle
both consume the arrays it returns, so bf16 workloads are rounded to
bf16-representable float32 values here, before either side sees them.

Workloads (sizes and distributions):

* ``pr1_ref``      fp32, 1 layer fwd; B=4, n ~ U{8..64}; d=64, H=2, dh=32;
                   W1, W2 ~ N(0, 0.02); X ~ N(0, 1); gaps Exp(60 s);
                   rab ~ N(0, 0.1) with 32 + 32 buckets; causal; N=64.
* ``academic``     bf16, 2 layers fwd; B=128, n ~ U{20..200}; d=64 (50-wide
                   item embeddings zero-padded); H=2, dh=32; X = E[ids] with
                   ids ~ Zipf(1.1) over a 3,706-row table E ~ N(0, 0.02);
                   N=200.  Synthetic stand-in for the public MovieLens-1M
                   catalogue size; no dataset is read.
* ``long_history`` bf16, 4 layers fwd; B=32, n from a power law
                   pdf ~ n^-1.2 on [256, 8192]; d=512, H=4, dh=128; N=8192.
* ``mfalcon``      bf16, 3 layers fwd; 16 users x (4,096 history + 1,024
                   candidates), microbatches of 256; d=512, H=4, dh=128;
                   N=5120; candidates share one request time per user.
* ``training``     bf16, 8 layers fwd+bwd; B=64, n ~ U{1024..8192}; d=1024,
                   H=8, dh=128; dY ~ N(0, 1); N=8192.

``sl_draws`` gives the Stochastic Length sampler its random inputs (uint32
keep-whole draws per sequence, uint32 ranking keys per row), uniform.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import os

import numpy as np


def round_to_bf16(a) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even) and
    return them as float32 (exactly representable in bf16).  Uses torch's
    CPU conversion, which rounds to nearest even."""
    import torch
    a = np.ascontiguousarray(a, dtype=np.float32)
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()


def normal_rows(seed: int, rows: int, cols: int, bf16: bool, std: float = 1.0,
                chunk: int = 8192) -> np.ndarray:
    """N(0, std^2) float32 matrix [rows, cols]; row-chunk k is drawn from the
    k-th child of SeedSequence(seed), so chunks fill in parallel threads and
    the result does not depend on the thread count."""
    import concurrent.futures as cf
    import torch
    out = np.empty((rows, cols), dtype=np.float32)
    nchunks = (rows + chunk - 1) // chunk
    children = np.random.SeedSequence(seed).spawn(max(nchunks, 1))

    def fill(k):
        r0, r1 = k * chunk, min(rows, (k + 1) * chunk)
        blk = out[r0:r1]
        np.random.default_rng(children[k]).standard_normal(size=blk.shape, dtype=np.float32, out=blk)
        if std != 1.0:
            blk *= np.float32(std)
        if bf16:
            t = torch.from_numpy(blk)
            t.copy_(t.to(torch.bfloat16).to(torch.float32))

    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
        list(ex.map(fill, range(nchunks)))
    return out


@dataclass
class Params:
    """One layer's weights as float32 arrays (bf16-representable when the
    workload is bf16).  Optional entries may be None."""
    W1: np.ndarray                      # [d, 4d]
    W2: np.ndarray                      # [d, d]
    rab_pos: Optional[np.ndarray]       # [H, P]
    rab_time: Optional[np.ndarray]      # [H, Bt]
    b1: Optional[np.ndarray] = None     # [4d]
    b2: Optional[np.ndarray] = None     # [d]
    gamma: Optional[np.ndarray] = None  # [d]
    beta: Optional[np.ndarray] = None   # [d]


@dataclass
class Workload:
    name: str
    dtype: str                  # "f32" or "bf16"
    d_model: int
    num_heads: int
    norm_N: float
    num_layers: int
    x: np.ndarray               # [T, d] float32
    seq_offsets: np.ndarray     # [B+1] int64
    timestamps: np.ndarray      # [T] int64 (seconds)
    num_targets: Optional[np.ndarray]  # [B] int32 or None
    params: List[Params]
    dy: Optional[np.ndarray] = None    # [T, d] upstream gradient (training)
    backward: bool = False
    microbatch: int = 0                # M-FALCON candidates per microbatch
    num_pos_buckets: int = 32
    num_time_buckets: int = 32
    ln_eps: float = 1e-5
    max_seq_len: int = 8192
    meta: Dict = field(default_factory=dict)

    @property
    def head_dim(self) -> int:
        return self.d_model // self.num_heads

    @property
    def B(self) -> int:
        return len(self.seq_offsets) - 1

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets)


# ----------------------------------------------------------------------------
# Building blocks
# ----------------------------------------------------------------------------

def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([np.zeros(1, np.int64), np.cumsum(lengths)]).astype(np.int64)


def draw_timestamps(rng, lengths, mean_gap: float = 60.0, start: int = 1_700_000_000):
    """Per sequence: a random start time, then strictly increasing times with
    gaps max(1, round(Exp(mean_gap))) seconds."""
    out = []
    for n in lengths:
        n = int(n)
        t0 = start + int(rng.integers(0, 10_000_000))
        gaps = np.maximum(1, np.rint(rng.exponential(mean_gap, size=max(n - 1, 0)))).astype(np.int64)
        out.append(t0 + np.concatenate([np.zeros(min(n, 1), np.int64), np.cumsum(gaps)]))
    return np.concatenate(out).astype(np.int64) if out else np.zeros(0, np.int64)


def draw_params(rng, d, H, P=32, Bt=32, w_std=0.02, rab_std=0.1, bf16=True,
                with_bias=False, with_affine=False) -> Params:
    r = round_to_bf16 if bf16 else (lambda a: np.asarray(a, np.float32))
    W1 = r(rng.normal(0.0, w_std, size=(d, 4 * d)).astype(np.float32))
    W2 = r(rng.normal(0.0, w_std, size=(d, d)).astype(np.float32))
    rab_pos = rng.normal(0.0, rab_std, size=(H, P)).astype(np.float32)
    rab_time = rng.normal(0.0, rab_std, size=(H, Bt)).astype(np.float32)
    p = Params(W1, W2, rab_pos, rab_time)
    if with_bias:
        p.b1 = r(rng.normal(0.0, w_std, size=(4 * d,)).astype(np.float32))
        p.b2 = r(rng.normal(0.0, w_std, size=(d,)).astype(np.float32))
    if with_affine:
        p.gamma = r((1.0 + rng.normal(0.0, 0.1, size=(d,))).astype(np.float32))
        p.beta = r(rng.normal(0.0, 0.1, size=(d,)).astype(np.float32))
    else:
        p.gamma = np.ones(d, np.float32)
        p.beta = np.zeros(d, np.float32)
    return p


def power_law_lengths(rng, B, alpha=1.2, lo=256, hi=8192):
    """Inverse-CDF draw from pdf ~ n^-alpha on [lo, hi], floored."""
    u = rng.random(B)
    a, b = lo ** (1.0 - alpha), hi ** (1.0 - alpha)
    n = (a + u * (b - a)) ** (1.0 / (1.0 - alpha))
    return np.clip(np.floor(n).astype(np.int64), lo, hi)


def zipf_ids(rng, size, s=1.1, rows=3706):
    """Item ids drawn from p(k) ~ k^-s on k = 1..rows (returned 0-based)."""
    k = np.arange(1, rows + 1, dtype=np.float64)
    p = k ** (-s)
    p /= p.sum()
    return rng.choice(rows, size=size, p=p)


# ----------------------------------------------------------------------------
# The five workloads
# ----------------------------------------------------------------------------

def _finish(name, dtype, d, H, N, layers, lengths, rng, seed, x=None, num_targets=None,
            backward=False, microbatch=0, timestamps=None, meta=None,
            with_bias=False, with_affine=False):
    bf16 = dtype == "bf16"
    lengths = np.asarray(lengths, dtype=np.int64)
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    if timestamps is None:
        timestamps = draw_timestamps(rng, lengths)
    if x is None:
        x = normal_rows(int(rng.integers(0, 2**62)), T, d, bf16)
    elif bf16:
        x = round_to_bf16(x)
    params = []
    for layer in range(layers):
        prng = np.random.default_rng(seed * 1000 + layer)
        params.append(draw_params(prng, d, H, bf16=bf16, with_bias=with_bias,
                                  with_affine=with_affine))
    dy = None
    if backward:
        dy = normal_rows(seed * 1000 + 999, T, d, bf16)
    return Workload(name=name, dtype=dtype, d_model=d, num_heads=H, norm_N=float(N),
                    num_layers=layers, x=x, seq_offsets=offs, timestamps=timestamps,
                    num_targets=num_targets, params=params, dy=dy, backward=backward,
                    microbatch=microbatch, meta=meta or {})


def pr1_ref(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    lengths = rng.integers(8, 65, size=4)
    return _finish("pr1_ref", "f32", 64, 2, 64, 1, lengths, rng, seed)


def academic(seed: int = 2, B: int = 128) -> Workload:
    rng = np.random.default_rng(seed)
    lengths = rng.integers(20, 201, size=B)
    T = int(lengths.sum())
    table = rng.normal(0.0, 0.02, size=(3706, 50)).astype(np.float32)
    ids = zipf_ids(rng, T)
    x = np.zeros((T, 64), np.float32)
    x[:, :50] = table[ids]
    return _finish("academic", "bf16", 64, 2, 200, 2, lengths, rng, seed, x=x,
                   meta={"item_ids": ids})


def long_history(seed: int = 3, B: int = 32) -> Workload:
    rng = np.random.default_rng(seed)
    lengths = power_law_lengths(rng, B)
    return _finish("long_history", "bf16", 512, 4, 8192, 4, lengths, rng, seed)


def mfalcon(seed: int = 4, users: int = 16, history: int = 4096, candidates: int = 1024,
            microbatch: int = 256) -> Workload:
    """Full-sequence view: each user is history + candidates with
    num_targets = candidates.  Candidates share the request time, one
    max(1, round(Exp(60))) gap after the last history event."""
    rng = np.random.default_rng(seed)
    lengths = np.full(users, history + candidates, dtype=np.int64)
    ts = []
    for _ in range(users):
        th = draw_timestamps(rng, [history])
        req = th[-1] + max(1, int(np.rint(rng.exponential(60.0))))
        ts.append(np.concatenate([th, np.full(candidates, req, np.int64)]))
    timestamps = np.concatenate(ts)
    num_targets = np.full(users, candidates, dtype=np.int32)
    return _finish("mfalcon", "bf16", 512, 4, 5120, 3, lengths, rng, seed,
                   num_targets=num_targets, timestamps=timestamps, microbatch=microbatch,
                   meta={"history": history, "candidates": candidates})


def training(seed: int = 5, B: int = 64, data_seed: Optional[int] = None) -> Workload:
    """`data_seed` (default: seed) draws lengths, inputs and timestamps;
    weights always come from `seed`, so data-parallel ranks share them."""
    rng = np.random.default_rng(seed if data_seed is None else data_seed)
    lengths = rng.integers(1024, 8193, size=B)
    w = _finish("training", "bf16", 1024, 8, 8192, 8, lengths, rng, seed, backward=True)
    if data_seed is not None and data_seed != seed:
        w.dy = normal_rows(data_seed * 1000 + 999, w.T, w.d_model, True)
    return w


WORKLOADS = {
    "pr1_ref": pr1_ref,
    "academic": academic,
    "long_history": long_history,
    "mfalcon": mfalcon,
    "training": training,
}


def custom(lengths, d=64, H=2, N=64.0, dtype="f32", layers=1, seed=11, num_targets=None,
           backward=False, with_bias=False, with_affine=False, x_std=1.0,
           timestamps=None, mean_gap=60.0) -> Workload:
    """A small workload with explicit lengths, used by tests for edge cases."""
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    T = int(lengths.sum())
    x = normal_rows(int(rng.integers(0, 2**62)), T, d, False, std=x_std)
    if timestamps is None:
        timestamps = draw_timestamps(rng, lengths, mean_gap=mean_gap)
    nt = None if num_targets is None else np.asarray(num_targets, dtype=np.int32)
    return _finish("custom", dtype, d, H, N, layers, lengths, rng, seed, x=x,
                   num_targets=nt, backward=backward, timestamps=timestamps,
                   with_bias=with_bias, with_affine=with_affine)


def subset(w: Workload, seqs) -> Workload:
    """The same workload restricted to the listed sequence indices (weights and
    normaliser unchanged)."""
    seqs = list(seqs)
    offs = w.seq_offsets
    rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in seqs]) if seqs else \
        np.zeros(0, np.int64)
    lengths = np.array([offs[b + 1] - offs[b] for b in seqs], dtype=np.int64)
    return Workload(name=w.name + "_subset", dtype=w.dtype, d_model=w.d_model,
                    num_heads=w.num_heads, norm_N=w.norm_N, num_layers=w.num_layers,
                    x=w.x[rows], seq_offsets=offsets_from_lengths(lengths),
                    timestamps=w.timestamps[rows],
                    num_targets=None if w.num_targets is None else w.num_targets[seqs],
                    params=w.params, dy=None if w.dy is None else w.dy[rows],
                    backward=w.backward, microbatch=w.microbatch,
                    num_pos_buckets=w.num_pos_buckets, num_time_buckets=w.num_time_buckets,
                    ln_eps=w.ln_eps, max_seq_len=w.max_seq_len, meta=dict(w.meta))


def sl_draws(seed: int, B: int, T: int, key_range: Optional[int] = None):
    """Random inputs of the Stochastic Length sampler: one uint32 keep-whole
    draw per sequence and one uint32 ranking key per input row.  A small
    ``key_range`` forces tied keys."""
    rng = np.random.default_rng(seed)
    keep = rng.integers(0, 1 << 32, size=B, dtype=np.uint64).astype(np.uint32)
    hi = (1 << 32) if key_range is None else int(key_range)
    keys = rng.integers(0, hi, size=T, dtype=np.uint64).astype(np.uint32)
    return keep, keys
