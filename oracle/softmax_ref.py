"""Plain fp64 CPU oracle of the softmax comparison attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path and never imports it; the product path must not call it.

The HSTU walkthrough (chenhuiyu.github.io, "generative-recommendation-16-hstu"),
section "No sequence-wise softmax", contrasts HSTU's pointwise SiLU
aggregation with the softmax attention of a standard Transformer: softmax
normalises every query's weights over the sequence positions, which the page
reports costs quality on the synthetic task (HR@10 0.0893 with pointwise SiLU
against 0.0617 with softmax).  The same paper's speed claim (the abstract on
mlsanity.com and the walkthrough's "The paper in 30 seconds": 5.3x-15.2x
faster than FlashAttention2-based Transformers at length 8,192) is about that
softmax attention.  This module states the softmax variant of equation (2):

    A_h(i, .) = softmax over the allowed keys j of S_h(i, j)
    O_h       = A_h V_h

Readings (the pages give no formula for the ablation): the score S_h is the
HSTU score unchanged, S_h(i, j) = Q_h(i) . K_h(j) + rab_pos[h][bp(i, j)] +
rab_time[h][bt(i, j)] with no 1/sqrt(dh) factor and the same buckets; the
mask is the same (causal, and M-FALCON candidates see the history and
themselves); masked pairs carry weight exactly 0; no 1/N scale (softmax
already normalises).  Every row has at least one allowed key (itself).
"""
from __future__ import annotations

import numpy as np

from .hstu_ref import F64, LayerConfig, _split, allowed_mask, bucket_ids


def masked_softmax_rows(S: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Row-wise softmax of S over the entries where mask holds; 0 elsewhere.
    The row maximum is subtracted first (the result does not depend on it)."""
    S = np.asarray(S, dtype=F64)
    x = np.where(mask, S, -np.inf)
    m = np.max(x, axis=1, keepdims=True)
    e = np.where(mask, np.exp(x - m), 0.0)
    return e / np.sum(e, axis=1, keepdims=True)


def softmax_attention_forward(g, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                              cfg: LayerConfig):
    """O[T, d] from G = U|V|Q|K [T, 4d] with softmax in place of SiLU/N."""
    g = np.asarray(g, dtype=F64)
    T, d4 = g.shape
    d = d4 // 4
    H = cfg.num_heads
    dh = d // H
    offs = np.asarray(seq_offsets, dtype=np.int64)
    ts = np.asarray(timestamps, dtype=np.int64)
    o = np.zeros((T, d))
    for b in range(len(offs) - 1):
        s, e = int(offs[b]), int(offs[b + 1])
        n = e - s
        if n == 0:
            continue
        m = 0 if num_targets is None else int(num_targets[b])
        mask = allowed_mask(n, m)
        bp, bt = bucket_ids(n, m, ts[s:e], cfg.num_pos_buckets, cfg.num_time_buckets)
        _, V, Q, K = _split(g[s:e], d)
        for hh in range(H):
            cs = slice(hh * dh, (hh + 1) * dh)
            bias = np.zeros((n, n))
            if rab_pos is not None:
                bias = bias + np.asarray(rab_pos[hh], F64)[bp]
            if rab_time is not None:
                bias = bias + np.asarray(rab_time[hh], F64)[bt]
            S = Q[:, cs] @ K[:, cs].T + bias
            o[s:e, cs] = masked_softmax_rows(S, mask) @ V[:, cs]
    return o
