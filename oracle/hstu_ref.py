"""Plain fp64 CPU oracle of one HSTU layer over jagged sequences.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path and never imports it; the product path must not call it.

What it computes (sources are the web pages about "Actions Speak Louder than
Words: Trillion-Parameter Sequential Transducers for Generative
Recommendations", arXiv 2402.17152):

* HSTU walkthrough (chenhuiyu.github.io, "generative-recommendation-16-hstu"),
  section "What an HSTU layer changes", equations (1)-(3):
      U, V, Q, K = Split(phi1(f1(X)))
      A(X) V     = phi2(Q K^T + rab^{p,t}) V
      Y          = f2(Norm(A(X) V) * U)
  with phi1 = phi2 = SiLU and rab^{p,t} a relative bias built from position
  and elapsed time.
* Same page, section "No sequence-wise softmax": SiLU is applied pointwise,
  nothing normalises across sequence positions, and the pooled value is then
  LayerNorm-ed.
* Same page, "Three more scaling components / Ragged kernels": computation is
  over the real (ragged) lengths; this oracle loops over sequences.
* "Sequential Transduction for Recommendation" (praveentn.live), section
  "What HSTU actually changed": the M-FALCON mask stops candidates attending
  to each other while they still see the user history.
* "Actions speak louder than words" course (yonasstephen.com), "Problem 2:
  position alone isn't enough" (bias from position and timestamps) and
  "Serving it: M-FALCON" (history work computed once and cached, candidates
  scored in microbatches against it).

Readings where the pages are silent:

* The pooled value is scaled by 1/N with N a per-configuration constant (not
  the sequence length); Q K^T carries no 1/sqrt(dh) factor.
* The layer output adds the input back: Y = f2(...) + X.
* Position bucket bp(i, j) = min(P-1, pos(i) - pos(j)) with pos(i) = min(i, h)
  where h is the history length (n minus the number of candidates).
* Time bucket bt(i, j) = 0 when dt = max(0, t_i - t_j) is 0, otherwise
  min(Bt-1, floor(log2 dt) + 1), computed with integer bit lengths.
* rab tables are per head: rab_pos[H, P], rab_time[H, Bt].
* allowed(i, j) = j <= i and (no candidates or j < h or j == i); masked pairs
  contribute exactly zero.
* LayerNorm is over all d = H*dh features of a token, biased variance,
  eps = 1e-5 by default, optional affine gamma/beta.
* Split order is U, V, Q, K as contiguous blocks of d columns; head k of a
  block is columns [k*dh, (k+1)*dh).
* Optional biases b1, b2 (absent in the stock workloads).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# Scalar building blocks
# ----------------------------------------------------------------------------

def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x)) (phi1 = phi2 = SiLU,
    HSTU walkthrough, "What an HSTU layer changes")."""
    x = np.asarray(x, dtype=F64)
    return x / (1.0 + np.exp(-x))


def silu_grad(x):
    """d/dx SiLU(x) = s(x) * (1 + x * (1 - s(x))) with s the logistic sigmoid."""
    x = np.asarray(x, dtype=F64)
    s = 1.0 / (1.0 + np.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def bit_length(v):
    """Exact integer bit length of non-negative int64 values (0 -> 0,
    1 -> 1, 2..3 -> 2, 4..7 -> 3, ...), without floating-point logarithms."""
    # binary search over the exponent: at each step, if v has a bit at or
    # above 2^k, count k bits and shift them out (integer arithmetic only)
    v = np.asarray(v, dtype=np.int64)
    out = np.zeros(v.shape, dtype=np.int64)
    for k in (32, 16, 8, 4, 2, 1):
        big = v >= (np.int64(1) << np.int64(k))
        out += big * np.int64(k)
        v = np.where(big, v >> np.int64(k), v)
    return out + (v > 0)


def time_bucket(dt, num_buckets):
    """Log2 time-gap bucket: 0 for a zero gap, else min(Bt-1, floor(log2 dt)+1).
    Negative gaps (never reached on allowed pairs) are clamped to 0."""
    dt = np.maximum(np.asarray(dt, dtype=np.int64), 0)
    return np.minimum(bit_length(dt), num_buckets - 1)


def pos_bucket(dpos, num_buckets):
    """Relative-position bucket: the clamped distance min(P-1, max(0, dpos))."""
    dpos = np.asarray(dpos, dtype=np.int64)
    return np.minimum(np.maximum(dpos, 0), num_buckets - 1)


# ----------------------------------------------------------------------------
# Parameters and configuration
# ----------------------------------------------------------------------------

@dataclass
class LayerParams:
    """One layer's parameters in fp64.  W1 is [d, 4d] (X @ W1), W2 is [d, d]."""
    W1: np.ndarray
    W2: np.ndarray
    rab_pos: Optional[np.ndarray] = None    # [H, P]
    rab_time: Optional[np.ndarray] = None   # [H, Bt]
    b1: Optional[np.ndarray] = None         # [4d]
    b2: Optional[np.ndarray] = None         # [d]
    gamma: Optional[np.ndarray] = None      # [d]
    beta: Optional[np.ndarray] = None       # [d]

    def as_f64(self) -> "LayerParams":
        f = lambda a: None if a is None else np.asarray(a, dtype=F64)
        return LayerParams(f(self.W1), f(self.W2), f(self.rab_pos), f(self.rab_time),
                           f(self.b1), f(self.b2), f(self.gamma), f(self.beta))


@dataclass
class LayerConfig:
    num_heads: int
    norm_N: float
    num_pos_buckets: int = 32
    num_time_buckets: int = 32
    ln_eps: float = 1e-5


# ----------------------------------------------------------------------------
# Masks and biases for one sequence
# ----------------------------------------------------------------------------

def allowed_mask(n: int, num_targets: int) -> np.ndarray:
    """allowed[i, j] for one sequence of n tokens whose last `num_targets`
    tokens are candidates (M-FALCON): causal, and candidates see the history
    and themselves but no other candidate."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    h = n - num_targets
    causal = j <= i
    if num_targets == 0:
        return causal
    return causal & ((j < h) | (j == i))


def bucket_ids(n: int, num_targets: int, timestamps: np.ndarray, P: int, Bt: int):
    """Position and time bucket ids [n, n] for one sequence."""
    h = n - num_targets
    idx = np.arange(n, dtype=np.int64)
    pos = np.minimum(idx, h)
    bp = pos_bucket(pos[:, None] - pos[None, :], P)
    ts = np.asarray(timestamps, dtype=np.int64)
    bt = time_bucket(ts[:, None] - ts[None, :], Bt)
    return bp, bt


def rab_bias(n, num_targets, timestamps, rab_pos_h, rab_time_h, P, Bt):
    """rab^{p,t}[i, j] = rab_pos[bp(i,j)] + rab_time[bt(i,j)] for one head."""
    bp, bt = bucket_ids(n, num_targets, timestamps, P, Bt)
    bias = np.zeros((n, n), dtype=F64)
    if rab_pos_h is not None:
        bias = bias + np.asarray(rab_pos_h, dtype=F64)[bp]
    if rab_time_h is not None:
        bias = bias + np.asarray(rab_time_h, dtype=F64)[bt]
    return bias


# ----------------------------------------------------------------------------
# Forward of one layer
# ----------------------------------------------------------------------------

@dataclass
class SeqCache:
    """Intermediates of one sequence kept for the backward pass."""
    x: np.ndarray
    pre: np.ndarray
    g: np.ndarray
    S: List[np.ndarray]
    A: List[np.ndarray]
    mask: np.ndarray
    bp: np.ndarray
    bt: np.ndarray
    o: np.ndarray
    ohat: np.ndarray
    rstd: np.ndarray
    lnout: np.ndarray
    z: np.ndarray


@dataclass
class LayerCache:
    seqs: List[SeqCache] = field(default_factory=list)


def _split(g: np.ndarray, d: int):
    return g[:, 0:d], g[:, d:2 * d], g[:, 2 * d:3 * d], g[:, 3 * d:4 * d]


def sequence_forward(x, timestamps, num_targets, p: LayerParams, cfg: LayerConfig,
                     keep: bool = False):
    """One layer on one sequence x[n, d].  Returns (y, cache or None)."""
    x = np.asarray(x, dtype=F64)
    n, d = x.shape
    H = cfg.num_heads
    dh = d // H
    P, Bt = cfg.num_pos_buckets, cfg.num_time_buckets

    # (1) U, V, Q, K = Split(SiLU(X W1 + b1))
    pre = x @ p.W1
    if p.b1 is not None:
        pre = pre + p.b1
    g = silu(pre)
    U, V, Q, K = _split(g, d)

    # (2) pointwise aggregated attention per head, masked, scaled by 1/N
    mask = allowed_mask(n, num_targets)
    bp, bt = bucket_ids(n, num_targets, timestamps, P, Bt)
    o = np.zeros((n, d), dtype=F64)
    S_list, A_list = [], []
    for hh in range(H):
        cs = slice(hh * dh, (hh + 1) * dh)
        bias = np.zeros((n, n), dtype=F64)
        if p.rab_pos is not None:
            bias = bias + p.rab_pos[hh][bp]
        if p.rab_time is not None:
            bias = bias + p.rab_time[hh][bt]
        S = Q[:, cs] @ K[:, cs].T + bias
        A = np.where(mask, silu(S), 0.0) / cfg.norm_N
        o[:, cs] = A @ V[:, cs]
        if keep:
            S_list.append(S)
            A_list.append(A)

    # (3) LayerNorm over the d features, gate by U, project, add residual
    mu = o.mean(axis=1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + cfg.ln_eps)
    ohat = (o - mu) * rstd
    ln = ohat
    if p.gamma is not None:
        ln = ln * p.gamma
    if p.beta is not None:
        ln = ln + p.beta
    z = ln * U
    y = z @ p.W2 + x
    if p.b2 is not None:
        y = y + p.b2
    cache = None
    if keep:
        cache = SeqCache(x, pre, g, S_list, A_list, mask, bp, bt, o, ohat, rstd, ln, z)
    return y, cache


def layer_forward(x, seq_offsets, timestamps, num_targets, params: LayerParams,
                  cfg: LayerConfig, keep: bool = False):
    """One layer over jagged values x[T, d] (sequences concatenated, bounds in
    seq_offsets[B+1]).  num_targets[B] may be None (plain causal)."""
    x = np.asarray(x, dtype=F64)
    p = params.as_f64()
    offs = np.asarray(seq_offsets, dtype=np.int64)
    ts = np.asarray(timestamps, dtype=np.int64)
    y = np.zeros_like(x)
    cache = LayerCache() if keep else None
    for b in range(len(offs) - 1):
        s, e = int(offs[b]), int(offs[b + 1])
        m = 0 if num_targets is None else int(num_targets[b])
        yb, cb = sequence_forward(x[s:e], ts[s:e], m, p, cfg, keep)
        y[s:e] = yb
        if keep:
            cache.seqs.append(cb)
    return y, cache


def stack_forward(x, seq_offsets, timestamps, num_targets, params_list: Sequence[LayerParams],
                  cfg: LayerConfig):
    """A stack of layers; no rounding between layers."""
    y = np.asarray(x, dtype=F64)
    for p in params_list:
        y, _ = layer_forward(y, seq_offsets, timestamps, num_targets, p, cfg)
    return y


# ----------------------------------------------------------------------------
# Backward of one layer (analytic chain rule of the forward above)
# ----------------------------------------------------------------------------

@dataclass
class LayerGrads:
    dW1: np.ndarray
    dW2: np.ndarray
    db1: np.ndarray
    db2: np.ndarray
    dgamma: np.ndarray
    dbeta: np.ndarray
    drab_pos: np.ndarray
    drab_time: np.ndarray


def sequence_backward(dy, c: SeqCache, p: LayerParams, cfg: LayerConfig, gr: LayerGrads):
    """Accumulates one sequence's parameter gradients into gr; returns dx."""
    dy = np.asarray(dy, dtype=F64)
    n, d = dy.shape
    H = cfg.num_heads
    dh = d // H
    U, V, Q, K = _split(c.g, d)

    # y = z W2 + b2 + x
    gr.dW2 += c.z.T @ dy
    gr.db2 += dy.sum(axis=0)
    dz = dy @ p.W2.T
    # z = ln * U
    dln = dz * U
    dU = dz * c.lnout
    # ln = ohat * gamma + beta
    gr.dbeta += dln.sum(axis=0)
    gr.dgamma += (dln * c.ohat).sum(axis=0)
    dohat = dln * p.gamma if p.gamma is not None else dln
    # ohat = (o - mu) * rstd, mean/var over the row
    do = c.rstd * (dohat - dohat.mean(axis=1, keepdims=True)
                   - c.ohat * (dohat * c.ohat).mean(axis=1, keepdims=True))

    dQ = np.zeros((n, d))
    dK = np.zeros((n, d))
    dV = np.zeros((n, d))
    for hh in range(H):
        cs = slice(hh * dh, (hh + 1) * dh)
        S, A = c.S[hh], c.A[hh]
        dA = do[:, cs] @ V[:, cs].T
        dV[:, cs] = A.T @ do[:, cs]
        dS = np.where(c.mask, dA * silu_grad(S), 0.0) / cfg.norm_N
        dQ[:, cs] = dS @ K[:, cs]
        dK[:, cs] = dS.T @ Q[:, cs]
        np.add.at(gr.drab_pos[hh], c.bp[c.mask], dS[c.mask])
        np.add.at(gr.drab_time[hh], c.bt[c.mask], dS[c.mask])

    dg = np.concatenate([dU, dV, dQ, dK], axis=1)
    dpre = dg * silu_grad(c.pre)
    gr.dW1 += c.x.T @ dpre
    gr.db1 += dpre.sum(axis=0)
    dx = dpre @ p.W1.T + dy
    return dx


def layer_backward(dy, seq_offsets, cache: LayerCache, params: LayerParams, cfg: LayerConfig):
    """Returns (dx, LayerGrads) for the jagged layer whose forward was run with keep=True."""
    p = params.as_f64()
    dy = np.asarray(dy, dtype=F64)
    d = dy.shape[1]
    H = cfg.num_heads
    gr = LayerGrads(np.zeros((d, 4 * d)), np.zeros((d, d)), np.zeros(4 * d), np.zeros(d),
                    np.zeros(d), np.zeros(d), np.zeros((H, cfg.num_pos_buckets)),
                    np.zeros((H, cfg.num_time_buckets)))
    offs = np.asarray(seq_offsets, dtype=np.int64)
    dx = np.zeros_like(dy)
    for b in range(len(offs) - 1):
        s, e = int(offs[b]), int(offs[b + 1])
        dx[s:e] = sequence_backward(dy[s:e], cache.seqs[b], p, cfg, gr)
    return dx, gr


def stack_forward_backward(x, seq_offsets, timestamps, num_targets, params_list, cfg, dy):
    """Forward through every layer keeping intermediates, then backward from
    dy.  Returns (y, dx, [LayerGrads per layer])."""
    caches = []
    h = np.asarray(x, dtype=F64)
    for p in params_list:
        h, c = layer_forward(h, seq_offsets, timestamps, num_targets, p, cfg, keep=True)
        caches.append(c)
    y = h
    g = np.asarray(dy, dtype=F64)
    grads = [None] * len(params_list)
    for li in range(len(params_list) - 1, -1, -1):
        g, grads[li] = layer_backward(g, seq_offsets, caches[li], params_list[li], cfg)
    return y, g, grads


# ----------------------------------------------------------------------------
# M-FALCON: history computed once and cached, candidates in microbatches
# ----------------------------------------------------------------------------

@dataclass
class HistoryCache:
    """Per layer: the history tokens' K and V (post-SiLU) and their timestamps."""
    K: List[np.ndarray]
    V: List[np.ndarray]
    timestamps: np.ndarray


def mfalcon_history(x_hist, timestamps_hist, params_list, cfg: LayerConfig):
    """Runs one user's history (a plain causal sequence) through the stack and
    caches each layer's K and V ("Serving it: M-FALCON": compute the history
    part once, cache it like attention KV caching)."""
    h = np.asarray(x_hist, dtype=F64)
    d = h.shape[1]
    Ks, Vs = [], []
    for p in params_list:
        pp = p.as_f64()
        pre = h @ pp.W1 + (pp.b1 if pp.b1 is not None else 0.0)
        g = silu(pre)
        Vs.append(g[:, d:2 * d].copy())
        Ks.append(g[:, 3 * d:4 * d].copy())
        h, _ = sequence_forward(h, timestamps_hist, 0, pp, cfg)
    return h, HistoryCache(Ks, Vs, np.asarray(timestamps_hist, dtype=np.int64))


def mfalcon_candidates(x_cand, timestamps_cand, cache: HistoryCache, params_list,
                       cfg: LayerConfig):
    """Scores one microbatch of candidates x_cand[c, d] against the cached
    history: each candidate attends to every history token and to itself,
    never to another candidate; its position is the history length."""
    h_len = cache.K[0].shape[0]
    xc = np.asarray(x_cand, dtype=F64)
    c_n, d = xc.shape
    H = cfg.num_heads
    dh = d // H
    P, Bt = cfg.num_pos_buckets, cfg.num_time_buckets
    tc = np.asarray(timestamps_cand, dtype=np.int64)
    th = cache.timestamps
    bp_hist = pos_bucket(h_len - np.arange(h_len, dtype=np.int64), P)            # [h]
    bt_hist = time_bucket(tc[:, None] - th[None, :], Bt)                        # [c, h]
    bp_self = pos_bucket(np.zeros(1, dtype=np.int64), P)[0]
    bt_self = time_bucket(np.zeros(1, dtype=np.int64), Bt)[0]
    for li, p in enumerate(params_list):
        pp = p.as_f64()
        pre = xc @ pp.W1 + (pp.b1 if pp.b1 is not None else 0.0)
        g = silu(pre)
        U, V, Q, K = _split(g, d)
        o = np.zeros((c_n, d))
        for hh in range(H):
            cs = slice(hh * dh, (hh + 1) * dh)
            rp = pp.rab_pos[hh] if pp.rab_pos is not None else np.zeros(P)
            rt = pp.rab_time[hh] if pp.rab_time is not None else np.zeros(Bt)
            S_hist = Q[:, cs] @ cache.K[li][:, cs].T + rp[bp_hist][None, :] + rt[bt_hist]
            s_self = (Q[:, cs] * K[:, cs]).sum(axis=1) + rp[bp_self] + rt[bt_self]
            o[:, cs] = (silu(S_hist) @ cache.V[li][:, cs]
                        + silu(s_self)[:, None] * V[:, cs]) / cfg.norm_N
        mu = o.mean(axis=1, keepdims=True)
        var = ((o - mu) ** 2).mean(axis=1, keepdims=True)
        ln = (o - mu) / np.sqrt(var + cfg.ln_eps)
        if pp.gamma is not None:
            ln = ln * pp.gamma
        if pp.beta is not None:
            ln = ln + pp.beta
        xc = (ln * U) @ pp.W2 + xc + (pp.b2 if pp.b2 is not None else 0.0)
    return xc


# ----------------------------------------------------------------------------
# Work counts used for reporting (algorithmic, masked pairs excluded)
# ----------------------------------------------------------------------------

def allowed_pairs(n: int, num_targets: int = 0) -> int:
    """|allowed| for one sequence: n(n+1)/2 causal; with m candidates
    h(h+1)/2 + m*h + m."""
    if num_targets == 0:
        return n * (n + 1) // 2
    h = n - num_targets
    return h * (h + 1) // 2 + num_targets * h + num_targets


def layer_flops_fwd(lengths, num_targets, d: int) -> int:
    """F_fwd = 10 T d^2 + 4 d sum_b |allowed_b| (projections + QK^T and AV)."""
    T = int(sum(lengths))
    pairs = sum(allowed_pairs(int(n), 0 if num_targets is None else int(m))
                for n, m in zip(lengths, num_targets if num_targets is not None
                                else [0] * len(lengths)))
    return 10 * T * d * d + 4 * d * pairs


# ----------------------------------------------------------------------------
# Single steps of the layer (for per-kernel parity).  Each restates one
# equation on jagged inputs; the CPU tests check that they compose back into
# layer_forward / layer_backward above.
# ----------------------------------------------------------------------------

def attention_forward(g, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                      cfg: LayerConfig):
    """Equation (2) alone: O[T, d] from G = U|V|Q|K [T, 4d]."""
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
            o[s:e, cs] = (np.where(mask, silu(S), 0.0) / cfg.norm_N) @ V[:, cs]
    return o


def ln_gate_forward(o, u, gamma, beta, eps):
    """Z = (LayerNorm(O) * gamma + beta) * U over each row; returns z, mean, rstd."""
    o = np.asarray(o, dtype=F64)
    mu = o.mean(axis=1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    ln = (o - mu) * rstd
    if gamma is not None:
        ln = ln * np.asarray(gamma, F64)
    if beta is not None:
        ln = ln + np.asarray(beta, F64)
    return ln * np.asarray(u, F64), mu[:, 0], rstd[:, 0]


def attention_backward(g, do, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                       cfg: LayerConfig):
    """Backward of attention_forward: returns dG [T, 4d] (U block zero),
    drab_pos [H, P], drab_time [H, Bt]."""
    g = np.asarray(g, dtype=F64)
    do = np.asarray(do, dtype=F64)
    T, d4 = g.shape
    d = d4 // 4
    H = cfg.num_heads
    dh = d // H
    P, Bt = cfg.num_pos_buckets, cfg.num_time_buckets
    offs = np.asarray(seq_offsets, dtype=np.int64)
    ts = np.asarray(timestamps, dtype=np.int64)
    dg = np.zeros((T, 4 * d))
    drp = np.zeros((H, P))
    drt = np.zeros((H, Bt))
    for b in range(len(offs) - 1):
        s, e = int(offs[b]), int(offs[b + 1])
        n = e - s
        m = 0 if num_targets is None else int(num_targets[b])
        mask = allowed_mask(n, m)
        bp, bt = bucket_ids(n, m, ts[s:e], P, Bt)
        _, V, Q, K = _split(g[s:e], d)
        for hh in range(H):
            cs = slice(hh * dh, (hh + 1) * dh)
            bias = np.zeros((n, n))
            if rab_pos is not None:
                bias = bias + np.asarray(rab_pos[hh], F64)[bp]
            if rab_time is not None:
                bias = bias + np.asarray(rab_time[hh], F64)[bt]
            S = Q[:, cs] @ K[:, cs].T + bias
            A = np.where(mask, silu(S), 0.0) / cfg.norm_N
            dA = do[s:e, cs] @ V[:, cs].T
            dS = np.where(mask, dA * silu_grad(S), 0.0) / cfg.norm_N
            dg[s:e, d + hh * dh:d + (hh + 1) * dh] = A.T @ do[s:e, cs]
            dg[s:e, 2 * d + hh * dh:2 * d + (hh + 1) * dh] = dS @ K[:, cs]
            dg[s:e, 3 * d + hh * dh:3 * d + (hh + 1) * dh] = dS.T @ Q[:, cs]
            np.add.at(drp[hh], bp[mask], dS[mask])
            np.add.at(drt[hh], bt[mask], dS[mask])
    return dg, drp, drt


def ln_gate_backward(dz, o, u, gamma, beta, eps):
    """Backward of ln_gate_forward: returns do, du, dgamma, dbeta."""
    dz = np.asarray(dz, F64)
    o = np.asarray(o, F64)
    u = np.asarray(u, F64)
    d = o.shape[1]
    gm = np.ones(d) if gamma is None else np.asarray(gamma, F64)
    bt = np.zeros(d) if beta is None else np.asarray(beta, F64)
    mu = o.mean(axis=1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    ohat = (o - mu) * rstd
    ln = ohat * gm + bt
    dln = dz * u
    du = dz * ln
    dohat = dln * gm
    do = rstd * (dohat - dohat.mean(axis=1, keepdims=True)
                 - ohat * (dohat * ohat).mean(axis=1, keepdims=True))
    return do, du, (dln * ohat).sum(axis=0), dln.sum(axis=0)
