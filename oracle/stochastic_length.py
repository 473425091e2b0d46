"""Plain CPU oracle of the Stochastic Length sampler (integer work, exact).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path and never imports it; the product path must not call it.

Source: HSTU walkthrough (chenhuiyu.github.io,
"generative-recommendation-16-hstu"), section "Three more scaling components /
Stochastic Length": training usually replaces a very long user history by a
shorter subsequence sampled from it and now and then keeps the whole history;
with alpha = 1.6 a history of 4,096 actions usually becomes 776 long, and the
quality cost is reported at 64%-84% sparsity.  The "Actions speak louder than
words" course (yonasstephen.com), "Problem 3: too slow at recommendation
scale", describes the same trick as subsampling long histories at random most
of the time because attention cost grows with the square of the length (the
walkthrough's section "Why user-level generative training saves a factor"
writes attention as O(N^2 d) for a maximum length N).

Readings where the pages are silent:

* Subsequence length L = floor(N^(alpha/2)) with N the maximum sequence
  length of the configuration.  This is the one reading that reproduces the
  printed pair: 4096^0.8 = 776.05 -> 776 (81% sparsity, inside 64%-84%).
* Only the history (the first h = n - num_targets positions) is sampled;
  candidate/target positions are always kept, after the history.
* A history with h <= L is kept whole.  A longer one is kept whole with
  probability L^2 / h^2, which bounds the expected attention cost of the
  history, E[h_kept^2] = 2 L^2 - L^4 / h^2 < 2 N^alpha: alpha is the exponent
  of the attention cost that is kept.
* The subsequence is a uniformly random L-subset of the history positions,
  kept in their original order (a causal sequence stays causal and its
  timestamps stay non-decreasing).

Random numbers are inputs, not drawn here: ``keep_draw[b]`` (uint32) decides
"keep whole" for sequence b, iff keep_draw[b] < (L*L / (h*h)) * 2^32 with the
quotient computed in fp64 (L*L and h*h exact integers, one correctly rounded
division); ``keys[t]`` (uint32, one per input row) rank the history positions:
the L positions with the smallest (key, position) pairs are selected, so i.i.d.
uniform keys give a uniform random subset and ties are broken by position.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

TWO32 = 4294967296.0


def subsequence_length(max_len: int, alpha: float) -> int:
    """L = floor(N^(alpha/2)) for maximum length N (walkthrough, "Stochastic
    Length": alpha = 1.6 maps 4,096 to 776)."""
    if max_len <= 0:
        return 0
    return int(math.floor(float(max_len) ** (alpha / 2.0)))


def keep_whole(h: int, L: int, draw: int) -> bool:
    """Whether a history of length h is kept whole, given its uint32 draw."""
    if h <= L:
        return True
    p = float(L * L) / float(h * h)
    return float(draw) < p * TWO32


def select_history(keys_b: np.ndarray, L: int) -> np.ndarray:
    """Positions (sorted) of the L smallest (key, position) pairs of one
    history.  The sort is a library primitive: lexsort orders by key, then by
    position."""
    h = len(keys_b)
    pos = np.arange(h, dtype=np.int64)
    order = np.lexsort((pos, keys_b.astype(np.int64)))
    return np.sort(order[:L]).astype(np.int64)


def sample(seq_offsets, num_targets: Optional[np.ndarray], L: int, keep_draw, keys
           ) -> Tuple[np.ndarray, np.ndarray]:
    """Stochastic Length over a jagged batch.

    Returns (new_offsets int64 [B+1], gather_index int64 [T']): output row r of
    the sampled batch is input row gather_index[r]; sequence b of the output
    owns rows [new_offsets[b], new_offsets[b+1]).
    """
    offs = np.asarray(seq_offsets, dtype=np.int64)
    B = len(offs) - 1
    keys = np.asarray(keys, dtype=np.uint32)
    keep_draw = np.asarray(keep_draw, dtype=np.uint32)
    new_offs = [0]
    idx = []
    for b in range(B):
        s, e = int(offs[b]), int(offs[b + 1])
        n = e - s
        m = int(num_targets[b]) if num_targets is not None else 0
        h = n - m
        if keep_whole(h, L, int(keep_draw[b])):
            rows = np.arange(s, e, dtype=np.int64)
        else:
            hist = s + select_history(keys[s:s + h], L)
            rows = np.concatenate([hist, np.arange(s + h, e, dtype=np.int64)])
        idx.append(rows)
        new_offs.append(new_offs[-1] + len(rows))
    gi = np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)
    return np.asarray(new_offs, dtype=np.int64), gi.astype(np.int64)


def gather(rows: np.ndarray, gather_index: np.ndarray) -> np.ndarray:
    """Output row r = input row gather_index[r] (embeddings, timestamps)."""
    return rows[gather_index]
