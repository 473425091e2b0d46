"""Pins of the fp64 oracle against facts other than itself (CPU only).

Each test ties one part of ``oracle/hstu_ref.py`` to something it does not
compute itself: hand-derived values, closed forms, brute-force scalar loops,
invariants (causality, jagged == padded, M-FALCON candidate independence),
finite differences, and an independent torch.float64 restatement with
autograd.  ``test_pins_catch_planted_mistakes`` plants mistakes in the oracle
and checks that these pins fail on them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import hstu_ref as R
from hstu_sequential_transducer_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def lp(p: W.Params) -> R.LayerParams:
    return R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)


def lcfg(w: W.Workload) -> R.LayerConfig:
    return R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)


# ----------------------------------------------------------------------------
# Bucket functions: hand table (tests/golden/buckets.txt)
# ----------------------------------------------------------------------------

def test_bucket_table_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "buckets.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) > 20
    for kind, v, b in rows:
        v, b = int(v), int(b)
        if kind == "time":
            got = int(R.time_bucket(np.array([v], np.int64), 32)[0])
        else:
            got = int(R.pos_bucket(np.array([v], np.int64), 32)[0])
        assert got == b, (kind, v, got, b)


def test_bucket_negative_gap_clamps_to_zero():
    assert int(R.time_bucket(np.array([-5], np.int64), 32)[0]) == 0


# ----------------------------------------------------------------------------
# SiLU closed forms
# ----------------------------------------------------------------------------

def test_silu_closed_forms():
    assert R.silu(0.0) == 0.0
    assert abs(R.silu(1.0) - math.e / (1.0 + math.e)) < 1e-15
    assert abs(R.silu(-1.0) - (-1.0 / (1.0 + math.e))) < 1e-15
    assert abs(R.silu(40.0) - 40.0) < 1e-12
    assert abs(R.silu(-40.0)) < 1e-15
    # derivative: s(0)(1 + 0) = 1/2 ; large x -> 1 ; central difference elsewhere
    assert abs(R.silu_grad(0.0) - 0.5) < 1e-15
    assert abs(R.silu_grad(40.0) - 1.0) < 1e-12
    for x in (-3.0, -1.2784645, 0.3, 2.5):
        h = 1e-6
        fd = (R.silu(x + h) - R.silu(x - h)) / (2 * h)
        assert abs(R.silu_grad(x) - fd) < 1e-9


# ----------------------------------------------------------------------------
# Hand-worked tiny layer (closed forms evaluated step by step)
# ----------------------------------------------------------------------------

def test_hand_worked_two_token_layer():
    """d = 2, H = 1, n = 2, N = 2.  W1 makes U = V = silu(x) blocks and
    Q = K = 0, so S is the bias alone:  S[i, j] = rp[bp] + rt[bt].
    With t = (100, 105): dt(1, 0) = 5 -> time bucket 3; dpos = 1 -> bucket 1.
    A = silu(S) / N on j <= i.  O = A V.  LayerNorm of a 2-vector [a, b] is
    [(a-b)/2, (b-a)/2] / sqrt((a-b)^2/4 + eps).  Y = (LN(O) * U) W2 + X with
    W2 = I."""
    x = np.array([[1.0, -2.0], [0.5, 3.0]])
    d = 2
    W1 = np.zeros((d, 4 * d))
    W1[:, 0:2] = np.eye(2)        # U = silu(x)
    W1[:, 2:4] = np.eye(2)        # V = silu(x)
    W2 = np.eye(2)
    rp = np.zeros((1, 32)); rp[0, 0] = 0.3; rp[0, 1] = -0.7
    rt = np.zeros((1, 32)); rt[0, 0] = 0.1; rt[0, 3] = 0.25
    p = R.LayerParams(W1, W2, rp, rt)
    cfg = R.LayerConfig(1, 2.0, 32, 32, 1e-5)
    y, _ = R.layer_forward(x, np.array([0, 2]), np.array([100, 105]), None, p, cfg)

    sil = lambda v: v / (1.0 + math.exp(-v))
    U = [[sil(v) for v in row] for row in x]
    V = U
    a00 = sil(0.3 + 0.1) / 2.0            # self: dpos 0, dt 0
    a10 = sil(-0.7 + 0.25) / 2.0          # dpos 1 -> bucket 1, dt 5 -> bucket 3
    a11 = a00
    O = [[a00 * V[0][0], a00 * V[0][1]],
         [a10 * V[0][0] + a11 * V[1][0], a10 * V[0][1] + a11 * V[1][1]]]
    expect = []
    for i in range(2):
        a, b = O[i]
        den = math.sqrt((a - b) ** 2 / 4.0 + 1e-5)
        ln = [(a - b) / 2.0 / den, (b - a) / 2.0 / den]
        expect.append([ln[0] * U[i][0] + x[i][0], ln[1] * U[i][1] + x[i][1]])
    np.testing.assert_allclose(y, np.array(expect), rtol=0, atol=1e-14)


def test_zero_w1_gives_residual_only():
    """W1 = 0 makes U = V = Q = K = silu(0) = 0, so Z = beta * 0 = 0 and
    Y = X + b2 exactly."""
    w = W.custom([5, 3], d=8, H=2, dtype="f32", with_bias=True, with_affine=True)
    p = lp(w.params[0])
    p.W1 = np.zeros_like(p.W1)
    p.b1 = None
    y, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, p, lcfg(w))
    np.testing.assert_array_equal(y, w.x.astype(np.float64) + p.b2.astype(np.float64))


def test_rab_only_special_case():
    """Q = K = 0 (their W1 blocks zero): S = rab only, A = silu(rab)/N on
    allowed pairs; checked entry by entry on n = 3."""
    w = W.custom([3], d=4, H=1, dtype="f32", N=3.0)
    p = lp(w.params[0])
    p.W1 = p.W1.copy()
    p.W1[:, 8:16] = 0.0
    ts = np.array([10, 13, 13 + 1000], np.int64)
    y, c = R.layer_forward(w.x, w.seq_offsets, ts, None, p, lcfg(w), keep=True)
    A = c.seqs[0].A[0]
    rp, rt = p.rab_pos[0].astype(np.float64), p.rab_time[0].astype(np.float64)
    sil = lambda v: v / (1.0 + math.exp(-v))
    # dt: (1,0)=3 -> 2; (2,0)=1003 -> 10; (2,1)=1000 -> 10; dpos 1, 2, 1
    expect = np.array([[sil(rp[0] + rt[0]), 0, 0],
                       [sil(rp[1] + rt[2]), sil(rp[0] + rt[0]), 0],
                       [sil(rp[2] + rt[10]), sil(rp[1] + rt[10]), sil(rp[0] + rt[0])]]) / 3.0
    np.testing.assert_allclose(A, expect, rtol=0, atol=1e-15)


def test_layernorm_closed_form_width_two_and_constant_rows():
    # width 2 (d = 2, H = 1)
    w = W.custom([4], d=2, H=1, dtype="f32")
    _, c = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, lp(w.params[0]), lcfg(w), keep=True)
    o = c.seqs[0].o
    a, b = o[:, 0], o[:, 1]
    den = np.sqrt((a - b) ** 2 / 4 + 1e-5)
    np.testing.assert_allclose(c.seqs[0].ohat, np.stack([(a - b) / 2 / den, (b - a) / 2 / den], 1),
                               rtol=0, atol=1e-13)
    # constant O rows: identical V columns with H = 1 -> LN(O) = beta, Y = X + (beta*U) W2
    w = W.custom([6], d=8, H=1, dtype="f32", with_affine=True)
    p = lp(w.params[0])
    p.W1 = p.W1.copy()
    p.W1[:, 8:16] = p.W1[:, 8:9]
    y, c = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, p, lcfg(w), keep=True)
    U = c.seqs[0].g[:, 0:8]
    np.testing.assert_allclose(y, w.x + (p.beta * U) @ p.W2, rtol=0, atol=1e-12)


def test_layernorm_row_statistics():
    w = W.custom([7, 9], d=16, H=4, dtype="f32")
    _, c = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, lp(w.params[0]), lcfg(w), keep=True)
    for s in c.seqs:
        var = s.o.var(axis=1)
        np.testing.assert_allclose(s.ohat.mean(axis=1), 0.0, atol=1e-12)
        np.testing.assert_allclose(s.ohat.var(axis=1), var / (var + 1e-5), rtol=1e-10)


# ----------------------------------------------------------------------------
# Brute force over all (i, j) pairs with scalar loops
# ----------------------------------------------------------------------------

def brute_force_layer(x, ts, m, p: R.LayerParams, H, N, eps):
    """Pure-Python scalar loops over tokens, features and pairs."""
    n, d = len(x), len(x[0])
    dh = d // H
    h_len = n - m
    sil = lambda v: v / (1.0 + math.exp(-v))
    G = [[0.0] * (4 * d) for _ in range(n)]
    for t in range(n):
        for c in range(4 * d):
            acc = p.b1[c] if p.b1 is not None else 0.0
            for k in range(d):
                acc += x[t][k] * p.W1[k][c]
            G[t][c] = sil(acc)
    y = []
    for i in range(n):
        o = [0.0] * d
        for hh in range(H):
            for j in range(n):
                ok = j <= i and (m == 0 or j < h_len or j == i)
                if not ok:
                    continue
                s = 0.0
                for e in range(dh):
                    s += G[i][2 * d + hh * dh + e] * G[j][3 * d + hh * dh + e]
                dp = min(i, h_len) - min(j, h_len)
                dt = ts[i] - ts[j]
                bt = 0
                while dt >= (1 << bt):
                    bt += 1
                s += p.rab_pos[hh][min(31, dp)] + p.rab_time[hh][min(31, bt)]
                a = sil(s) / N
                for e in range(dh):
                    o[hh * dh + e] += a * G[j][d + hh * dh + e]
        mu = sum(o) / d
        var = sum((v - mu) ** 2 for v in o) / d
        z = [((o[k] - mu) / math.sqrt(var + eps) * p.gamma[k] + p.beta[k]) * G[i][k] for k in range(d)]
        y.append([sum(z[k] * p.W2[k][c] for k in range(d)) + x[i][c] + (p.b2[c] if p.b2 is not None else 0.0)
                  for c in range(d)])
    return np.array(y)


@pytest.mark.parametrize("lengths,targets", [([7, 1, 12], None), ([9, 6], [3, 1]), ([5], [5])])
def test_brute_force_all_pairs(lengths, targets):
    w = W.custom(lengths, d=8, H=2, dtype="f32", N=7.0, num_targets=targets, with_bias=True,
                 with_affine=True, mean_gap=400.0)
    p = lp(w.params[0]).as_f64()
    y, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, p, lcfg(w))
    for b in range(w.B):
        s, e = w.seq_offsets[b], w.seq_offsets[b + 1]
        m = 0 if targets is None else targets[b]
        yb = brute_force_layer(w.x[s:e].astype(np.float64).tolist(), w.timestamps[s:e].tolist(), m,
                               p, w.num_heads, w.norm_N, w.ln_eps)
        np.testing.assert_allclose(y[s:e], yb, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# Zero rab == bare pointwise formula
# ----------------------------------------------------------------------------

def test_zero_rab_equals_bare_formula():
    w = W.custom([11, 4], d=8, H=2, dtype="f32")
    p = lp(w.params[0])
    p0 = R.LayerParams(p.W1, p.W2, np.zeros_like(p.rab_pos), np.zeros_like(p.rab_time),
                       gamma=p.gamma, beta=p.beta)
    pn = R.LayerParams(p.W1, p.W2, None, None, gamma=p.gamma, beta=p.beta)
    cfg = lcfg(w)
    _, c0 = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, p0, cfg, keep=True)
    _, cn = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, pn, cfg, keep=True)
    for b in range(w.B):
        s, e = w.seq_offsets[b], w.seq_offsets[b + 1]
        X = w.x[s:e].astype(np.float64)
        pre = X @ p.W1.astype(np.float64)
        G = pre * (1 / (1 + np.exp(-pre)))
        n = e - s
        Mc = np.tril(np.ones((n, n)))
        for hh in range(2):
            cs = slice(16 + hh * 4, 16 + hh * 4 + 4)
            ks = slice(24 + hh * 4, 24 + hh * 4 + 4)
            vs = slice(8 + hh * 4, 8 + hh * 4 + 4)
            QK = np.einsum("ie,je->ij", G[:, cs], G[:, ks])
            O = (QK * (1 / (1 + np.exp(-QK))) * Mc / w.norm_N) @ G[:, vs]
            np.testing.assert_allclose(c0.seqs[b].o[:, hh * 4:(hh + 1) * 4], O, rtol=0, atol=1e-14)
            np.testing.assert_allclose(cn.seqs[b].o[:, hh * 4:(hh + 1) * 4], O, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# Causality and jagged independence
# ----------------------------------------------------------------------------

def test_causality_perturbation():
    w = W.custom([13], d=8, H=2, dtype="f32")
    p, cfg = lp(w.params[0]), lcfg(w)
    y, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, p, cfg)
    for i in (0, 5, 11):
        x2 = w.x.copy()
        x2[i + 1:] = np.random.default_rng(i).normal(size=x2[i + 1:].shape)
        ts2 = w.timestamps.copy()
        ts2[i + 1:] += 12345
        y2, _ = R.layer_forward(x2, w.seq_offsets, ts2, None, p, cfg)
        np.testing.assert_array_equal(y[:i + 1], y2[:i + 1])
        assert np.abs(y[i + 1:] - y2[i + 1:]).max() > 1e-3


def test_jagged_sequences_are_independent():
    w = W.custom([6, 1, 9, 3], d=8, H=2, dtype="f32", num_targets=[2, 0, 4, 1])
    p, cfg = lp(w.params[0]), lcfg(w)
    y, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, p, cfg)
    for b in range(w.B):
        s, e = w.seq_offsets[b], w.seq_offsets[b + 1]
        yb, _ = R.layer_forward(w.x[s:e], np.array([0, e - s]), w.timestamps[s:e],
                                w.num_targets[b:b + 1], p, cfg)
        np.testing.assert_array_equal(y[s:e], yb)


# ----------------------------------------------------------------------------
# Independent torch.float64 restatement (padded dense batch + autograd)
# ----------------------------------------------------------------------------

def torch_padded_layer(w: W.Workload, p: W.Params, x=None):
    """Padded [B, n_max, d] formulation with explicit masks; buckets through
    torch.frexp (exact below 2^53) rather than integer bit lengths."""
    dt = torch.float64
    B, d, H = w.B, w.d_model, w.num_heads
    dh = d // H
    lens = w.lengths.tolist()
    nmax = max(lens) if lens else 0
    X = torch.zeros(B, nmax, d, dtype=dt)
    Ts = torch.zeros(B, nmax, dtype=torch.int64)
    xs = torch.as_tensor(w.x, dtype=dt) if x is None else x
    for b in range(B):
        s, e = int(w.seq_offsets[b]), int(w.seq_offsets[b + 1])
        X[b, :e - s] = xs[s:e]
        Ts[b, :e - s] = torch.as_tensor(w.timestamps[s:e])
    P = {k: (None if getattr(p, k) is None else torch.tensor(getattr(p, k), dtype=dt, requires_grad=True))
         for k in ("W1", "W2", "rab_pos", "rab_time", "b1", "b2", "gamma", "beta")}
    pre = X @ P["W1"] + (P["b1"] if P["b1"] is not None else 0)
    G = torch.nn.functional.silu(pre)
    U, V, Q, K = G.split(d, dim=-1)
    idx = torch.arange(nmax)
    valid = torch.stack([idx < n for n in lens]) if lens else torch.zeros(0, nmax, dtype=torch.bool)
    m = torch.tensor([0 if w.num_targets is None else int(w.num_targets[b]) for b in range(B)])
    hl = torch.tensor(lens) - m
    ii, jj = idx[:, None], idx[None, :]
    allow = (jj <= ii)[None] & valid[:, None, :] & valid[:, :, None]
    allow = allow & ((m[:, None, None] == 0) | (jj[None] < hl[:, None, None]) | (ii == jj)[None])
    pos = torch.minimum(idx[None], hl[:, None])
    dp = (pos[:, :, None] - pos[:, None, :]).clamp(0, 31)
    gap = (Ts[:, :, None] - Ts[:, None, :]).clamp(min=0).to(dt)
    _, ex = torch.frexp(gap)
    bt = torch.where(gap > 0, ex.to(torch.int64), torch.zeros_like(ex, dtype=torch.int64)).clamp(max=31)
    Qh = Q.view(B, nmax, H, dh).transpose(1, 2)
    Kh = K.view(B, nmax, H, dh).transpose(1, 2)
    Vh = V.view(B, nmax, H, dh).transpose(1, 2)
    S = Qh @ Kh.transpose(-1, -2)
    S = S + P["rab_pos"][:, dp].permute(1, 0, 2, 3) + P["rab_time"][:, bt].permute(1, 0, 2, 3)
    A = torch.where(allow[:, None], torch.nn.functional.silu(S), torch.zeros((), dtype=dt)) / w.norm_N
    O = (A @ Vh).transpose(1, 2).reshape(B, nmax, d)
    Ln = torch.nn.functional.layer_norm(O, (d,), P["gamma"], P["beta"], eps=w.ln_eps)
    Y = (Ln * U) @ P["W2"] + X + (P["b2"] if P["b2"] is not None else 0)
    out = torch.cat([Y[b, :lens[b]] for b in range(B)]) if B else Y.reshape(0, d)
    return out, P


@pytest.mark.parametrize("targets", [None, [2, 0, 3]])
def test_torch_autograd_cross_check(targets):
    w = W.custom([5, 8, 6], d=8, H=2, dtype="f32", N=5.0, num_targets=targets, with_bias=True,
                 with_affine=True, backward=True, mean_gap=300.0)
    p = w.params[0]
    xt = torch.tensor(w.x, dtype=torch.float64, requires_grad=True)
    yt, P = torch_padded_layer(w, p, xt)
    (yt * torch.tensor(w.dy, dtype=torch.float64)).sum().backward()
    cfg = lcfg(w)
    y, cache = R.layer_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, lp(p), cfg, keep=True)
    dx, g = R.layer_backward(w.dy, w.seq_offsets, cache, lp(p), cfg)
    np.testing.assert_allclose(y, yt.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=0, atol=1e-11)
    for name, ours in (("W1", g.dW1), ("W2", g.dW2), ("b1", g.db1), ("b2", g.db2),
                       ("gamma", g.dgamma), ("beta", g.dbeta), ("rab_pos", g.drab_pos),
                       ("rab_time", g.drab_time)):
        np.testing.assert_allclose(ours, P[name].grad.numpy(), rtol=0, atol=1e-11, err_msg=name)


# ----------------------------------------------------------------------------
# Finite differences for every gradient
# ----------------------------------------------------------------------------

def test_gradients_central_differences():
    w = W.custom([4, 3], d=4, H=2, dtype="f32", N=3.0, num_targets=[1, 0], with_bias=True,
                 with_affine=True, backward=True, mean_gap=500.0)
    p = lp(w.params[0]).as_f64()
    cfg = lcfg(w)
    dy = w.dy.astype(np.float64)
    _, cache = R.layer_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, p, cfg, keep=True)
    dx, g = R.layer_backward(dy, w.seq_offsets, cache, p, cfg)

    def loss(x=None, **over):
        q = R.LayerParams(**{k: over.get(k, getattr(p, k)) for k in
                             ("W1", "W2", "rab_pos", "rab_time", "b1", "b2", "gamma", "beta")})
        y, _ = R.layer_forward(w.x if x is None else x, w.seq_offsets, w.timestamps,
                               w.num_targets, q, cfg)
        return float((y * dy).sum())

    h = 1e-6
    rng = np.random.default_rng(0)

    def check(name, analytic, base, as_x=False):
        flat = base.reshape(-1)
        picks = rng.choice(flat.size, size=min(12, flat.size), replace=False)
        for k in picks:
            a = base.copy().reshape(-1); a[k] += h
            b = base.copy().reshape(-1); b[k] -= h
            a, b = a.reshape(base.shape), b.reshape(base.shape)
            fa = loss(x=a) if as_x else loss(**{name: a})
            fb = loss(x=b) if as_x else loss(**{name: b})
            fd = (fa - fb) / (2 * h)
            an = analytic.reshape(-1)[k]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, k, fd, an)

    check("x", dx, w.x.astype(np.float64), as_x=True)
    for name, an in (("W1", g.dW1), ("W2", g.dW2), ("b1", g.db1), ("b2", g.db2),
                     ("gamma", g.dgamma), ("beta", g.dbeta), ("rab_pos", g.drab_pos),
                     ("rab_time", g.drab_time)):
        check(name, an, getattr(p, name))


# ----------------------------------------------------------------------------
# M-FALCON: candidate independence, microbatch split, reduction to causal
# ----------------------------------------------------------------------------

def _mf_workload(users=2, hist=9, cand=6, d=8, H=2):
    rng = np.random.default_rng(7)
    lengths = [hist + cand] * users
    ts = []
    for _ in range(users):
        th = W.draw_timestamps(rng, [hist], mean_gap=200.0)
        ts.append(np.concatenate([th, np.full(cand, th[-1] + 77, np.int64)]))
    return W.custom(lengths, d=d, H=H, dtype="f32", N=float(hist + cand), num_targets=[cand] * users,
                    timestamps=np.concatenate(ts), layers=2, with_affine=True)


def test_mfalcon_cached_equals_target_mask_and_is_split_invariant():
    w = _mf_workload()
    cfg = lcfg(w)
    plist = [lp(p) for p in w.params]
    y_full = R.stack_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, plist, cfg)
    hist, cand = 9, 6
    for b in range(w.B):
        s = w.seq_offsets[b]
        xh, th = w.x[s:s + hist], w.timestamps[s:s + hist]
        xc, tc = w.x[s + hist:s + hist + cand], w.timestamps[s + hist:s + hist + cand]
        yh, cache = R.mfalcon_history(xh, th, plist, cfg)
        np.testing.assert_allclose(yh, y_full[s:s + hist], rtol=0, atol=1e-12)
        for mb in (1, 2, 4, 6):
            outs = [R.mfalcon_candidates(xc[k:k + mb], tc[k:k + mb], cache, plist, cfg)
                    for k in range(0, cand, mb)]
            np.testing.assert_allclose(np.concatenate(outs), y_full[s + hist:s + hist + cand],
                                       rtol=0, atol=1e-12)


def test_mfalcon_candidate_independence():
    w = _mf_workload(users=1)
    cfg = lcfg(w)
    plist = [lp(p) for p in w.params]
    y = R.stack_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, plist, cfg)
    hist, cand = 9, 6
    # alter other candidates
    x2 = w.x.copy()
    x2[hist + 1:] = np.random.default_rng(1).normal(size=x2[hist + 1:].shape)
    y2 = R.stack_forward(x2, w.seq_offsets, w.timestamps, w.num_targets, plist, cfg)
    np.testing.assert_allclose(y2[:hist + 1], y[:hist + 1], rtol=0, atol=1e-13)
    # permute candidates
    perm = np.r_[np.arange(hist), hist + np.random.default_rng(2).permutation(cand)]
    y3 = R.stack_forward(w.x[perm], w.seq_offsets, w.timestamps[perm], w.num_targets, plist, cfg)
    np.testing.assert_allclose(y3, y[perm], rtol=0, atol=1e-13)
    # remove all candidates but one
    keep = np.r_[np.arange(hist), hist + 3]
    y4 = R.stack_forward(w.x[keep], np.array([0, hist + 1]), w.timestamps[keep],
                         np.array([1], np.int32), plist, cfg)
    np.testing.assert_allclose(y4, y[keep], rtol=0, atol=1e-13)


def test_one_target_equals_causal():
    w = W.custom([10, 5], d=8, H=2, dtype="f32", num_targets=[1, 1])
    p, cfg = lp(w.params[0]), lcfg(w)
    y1, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets, p, cfg)
    y0, _ = R.layer_forward(w.x, w.seq_offsets, w.timestamps, None, p, cfg)
    np.testing.assert_array_equal(y1, y0)


# ----------------------------------------------------------------------------
# Work counts
# ----------------------------------------------------------------------------

def test_allowed_pair_counts_match_masks():
    for n, m in ((1, 0), (9, 0), (9, 3), (9, 9), (5, 1)):
        assert R.allowed_pairs(n, m) == int(R.allowed_mask(n, m).sum())


# ----------------------------------------------------------------------------
# The pins bite: plant mistakes in the oracle and see at least one pin fail
# ----------------------------------------------------------------------------

MUTANTS = {
    "time_bucket_off_by_one": ("time_bucket",
                               lambda orig: (lambda dt, nb: np.minimum(orig(dt, nb) + 1, nb - 1))),
    "pos_bucket_unclamped_low": ("pos_bucket",
                                 lambda orig: (lambda dp, nb: np.minimum(np.abs(dp) + 1, nb - 1))),
    "silu_as_sigmoid": ("silu", lambda orig: (lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, float))))),
    "silu_grad_drops_term": ("silu_grad",
                             lambda orig: (lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, float))))),
    "mask_not_causal": ("allowed_mask", lambda orig: (lambda n, m: np.ones((n, n), bool))),
    "mask_candidates_see_each_other": ("allowed_mask",
                                       lambda orig: (lambda n, m: orig(n, 0))),
}


def _pin_suite():
    """The pins re-run against a (possibly mutated) oracle; returns the
    number of pins that failed."""
    fails = 0
    for fn in (test_bucket_table_golden, test_silu_closed_forms, test_hand_worked_two_token_layer,
               test_rab_only_special_case, lambda: test_torch_autograd_cross_check(None),
               lambda: test_torch_autograd_cross_check([2, 0, 3]),
               test_causality_perturbation, test_zero_rab_equals_bare_formula,
               test_mfalcon_candidate_independence):
        try:
            fn()
        except AssertionError:
            fails += 1
        except Exception:
            fails += 1
    return fails


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    attr, make = MUTANTS[mutant]
    orig = getattr(R, attr)
    monkeypatch.setattr(R, attr, make(orig))
    assert _pin_suite() > 0, f"no pin caught mutant {mutant}"


# ----------------------------------------------------------------------------
# Single-step oracle functions compose back into the pinned layer
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("targets", [None, [3, 0, 6]])
def test_step_functions_compose_to_layer(targets):
    w = W.custom([9, 4, 6], d=16, H=2, dtype="f32", N=6.0, num_targets=targets, with_bias=True,
                 with_affine=True, backward=True, mean_gap=250.0)
    p = lp(w.params[0]).as_f64()
    cfg = lcfg(w)
    nt = w.num_targets
    y, cache = R.layer_forward(w.x, w.seq_offsets, w.timestamps, nt, p, cfg, keep=True)
    dx, gr = R.layer_backward(w.dy, w.seq_offsets, cache, p, cfg)
    x = w.x.astype(np.float64)
    d = 16
    pre = x @ p.W1 + p.b1
    g = R.silu(pre)
    o = R.attention_forward(g, w.seq_offsets, w.timestamps, nt, p.rab_pos, p.rab_time, cfg)
    z, mu, rstd = R.ln_gate_forward(o, g[:, :d], p.gamma, p.beta, cfg.ln_eps)
    y2 = z @ p.W2 + p.b2 + x
    np.testing.assert_allclose(y2, y, rtol=0, atol=1e-13)
    dy = w.dy.astype(np.float64)
    dz = dy @ p.W2.T
    do, du, dgam, dbet = R.ln_gate_backward(dz, o, g[:, :d], p.gamma, p.beta, cfg.ln_eps)
    dg, drp, drt = R.attention_backward(g, do, w.seq_offsets, w.timestamps, nt, p.rab_pos,
                                        p.rab_time, cfg)
    dg[:, :d] = du
    dpre = dg * R.silu_grad(pre)
    np.testing.assert_allclose(dpre @ p.W1.T + dy, dx, rtol=0, atol=1e-12)
    np.testing.assert_allclose(x.T @ dpre, gr.dW1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dgam, gr.dgamma, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dbet, gr.dbeta, rtol=0, atol=1e-12)
    np.testing.assert_allclose(drp, gr.drab_pos, rtol=0, atol=1e-12)
    np.testing.assert_allclose(drt, gr.drab_time, rtol=0, atol=1e-12)
