"""Pins of the softmax comparison oracle (oracle/softmax_ref.py), CPU only.

Each pin holds the oracle to something other than itself: a library softmax,
closed forms (a single allowed key copies its value; equal scores average the
values; a two-token case worked by hand), softmax's invariance to a shift of
every score, causality and the M-FALCON candidates' independence.  Planted
mistakes in the oracle must each fail at least one pin.
"""
import numpy as np
import pytest
from scipy.special import softmax as scipy_softmax

from oracle import hstu_ref as R
from oracle import softmax_ref as SR
from hstu_sequential_transducer_b200 import workloads as W


def _case(lengths, nt=None, d=16, H=2, seed=3):
    rng = np.random.default_rng(seed)
    w = W.custom(lengths, d=d, H=H, dtype="f32", N=64.0, num_targets=nt, seed=seed)
    g = rng.normal(0, 0.7, size=(w.T, 4 * d))
    p = w.params[0]
    cfg = R.LayerConfig(H, 64.0)
    return w, g, p, cfg


def _fwd(w, g, p, cfg, fn=None):
    fn = fn or SR.softmax_attention_forward
    return fn(g, w.seq_offsets, w.timestamps, w.num_targets, p.rab_pos, p.rab_time, cfg)


def test_rows_match_a_library_softmax():
    rng = np.random.default_rng(0)
    S = rng.normal(0, 3, size=(9, 9))
    mask = R.allowed_mask(9, 3)
    A = SR.masked_softmax_rows(S, mask)
    for i in range(9):
        np.testing.assert_allclose(A[i, mask[i]], scipy_softmax(S[i, mask[i]]), rtol=1e-14)
        assert np.all(A[i, ~mask[i]] == 0.0)
    np.testing.assert_allclose(A.sum(axis=1), 1.0, rtol=1e-14)


def test_first_token_copies_its_value():
    """Token 0 of a sequence sees only itself: its weight is 1."""
    w, g, p, cfg = _case([5, 1, 7])
    o = _fwd(w, g, p, cfg)
    d = w.d_model
    for s in w.seq_offsets[:-1]:
        np.testing.assert_allclose(o[s], g[s, d:2 * d], rtol=1e-14, atol=1e-14)


def test_equal_scores_average_the_allowed_values():
    """Q = 0 and no rab: every allowed key has the same score, so each output
    is the plain mean of the values it may see."""
    w, g, p, cfg = _case([6, 4], nt=[0, 2], d=8, H=1)
    d = w.d_model
    g[:, 2 * d:3 * d] = 0.0
    o = SR.softmax_attention_forward(g, w.seq_offsets, w.timestamps, w.num_targets, None, None, cfg)
    for b in range(2):
        s, e = int(w.seq_offsets[b]), int(w.seq_offsets[b + 1])
        n = e - s
        mask = R.allowed_mask(n, int(w.num_targets[b]))
        V = g[s:e, d:2 * d]
        for i in range(n):
            np.testing.assert_allclose(o[s + i], V[mask[i]].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_two_token_case_by_hand():
    """n = 2, one head of width 2, integer-valued G; position buckets 0 and 1,
    time gap 3 s (bucket 2, since 3 has bit length 2)."""
    d = 2
    g = np.zeros((2, 8))
    g[:, d:2 * d] = [[1.0, -2.0], [3.0, 5.0]]        # V
    g[:, 2 * d:3 * d] = [[1.0, 0.0], [1.0, 2.0]]     # Q
    g[:, 3 * d:4 * d] = [[2.0, 1.0], [0.0, 1.0]]     # K
    rp = np.zeros((1, 32))
    rt = np.zeros((1, 32))
    rp[0, 0], rp[0, 1] = 0.5, -1.0
    rt[0, 0], rt[0, 2] = 0.25, 1.5
    cfg = R.LayerConfig(1, 1.0)
    o = SR.softmax_attention_forward(g, np.array([0, 2]), np.array([10, 13]), None, rp, rt, cfg)
    # row 1: s10 = q1.k0 + rp[1] + rt[2] = 4 - 1 + 1.5 = 4.5 ; s11 = q1.k1 + rp[0] + rt[0] = 2.75
    e0, e1 = np.exp(4.5), np.exp(2.75)
    want1 = (e0 * np.array([1.0, -2.0]) + e1 * np.array([3.0, 5.0])) / (e0 + e1)
    np.testing.assert_allclose(o[0], [1.0, -2.0], rtol=1e-15)
    np.testing.assert_allclose(o[1], want1, rtol=1e-14)


def test_shift_of_every_score_changes_nothing():
    w, g, p, cfg = _case([9, 12], nt=[0, 4])
    o = _fwd(w, g, p, cfg)
    o2 = SR.softmax_attention_forward(g, w.seq_offsets, w.timestamps, w.num_targets,
                                      np.asarray(p.rab_pos, np.float64) + 3.25,
                                      np.asarray(p.rab_time, np.float64) - 1.5, cfg)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)


def test_causality_and_candidate_independence():
    w, g, p, cfg = _case([10], nt=[4])
    o = _fwd(w, g, p, cfg)
    g2 = g.copy()
    g2[7] += 1.0            # a candidate: no other token may see it
    o2 = _fwd(w, g2, p, cfg)
    keep = [i for i in range(10) if i != 7]
    np.testing.assert_array_equal(o2[keep], o[keep])
    g3 = g.copy()
    g3[4] += 1.0            # history token 4: tokens before it are unchanged
    o3 = _fwd(w, g3, p, cfg)
    np.testing.assert_array_equal(o3[:4], o[:4])


# ----------------------------------------------------------------------------
# Planted mistakes: each must fail one of the pins above
# ----------------------------------------------------------------------------

_softmax = SR.masked_softmax_rows


def _mut_no_mask(S, mask):
    return _softmax(S, np.ones_like(mask))


def _mut_unnormalised(S, mask):
    x = np.where(mask, S, -np.inf)
    return np.where(mask, np.exp(x - np.max(x, axis=1, keepdims=True)), 0.0)


def _mut_transposed(S, mask):
    return _softmax(S, mask).T


def _mut_column_softmax(S, mask):
    return _softmax(S.T, mask.T).T


@pytest.mark.parametrize("mutant", [_mut_no_mask, _mut_unnormalised, _mut_transposed,
                                    _mut_column_softmax])
def test_planted_mistakes_fail_a_pin(monkeypatch, mutant):
    monkeypatch.setattr(SR, "masked_softmax_rows", mutant)
    pins = [test_rows_match_a_library_softmax, test_first_token_copies_its_value,
            test_equal_scores_average_the_allowed_values, test_two_token_case_by_hand,
            test_causality_and_candidate_independence]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1
