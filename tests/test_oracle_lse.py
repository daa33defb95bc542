"""Pins of the oracle's per-row log-sum-exp (routed_attention_row_lse): a single
key gives its own logit, n identical keys add log n, the softmax weights it
normalises sum to 1 and reproduce routed_attention_row's output, it is invariant
to the key order, and a planted log2 in place of the natural log fails."""
import math

import numpy as np

from oracle import msa_oracle as O


def _row(rng, d=64, M=50, Lc=9, qi=6):
    return (rng.standard_normal(d), qi, 1000, 10000.0, rng.standard_normal((M, d)),
            rng.standard_normal((M, d)), rng.standard_normal((Lc, d)), rng.standard_normal((Lc, d)))


def test_single_key_is_its_logit():
    rng = np.random.default_rng(0)
    d = 64
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    # no memory keys, local index 0: the only key is local key 0 at position k_off
    lse = O.routed_attention_row_lse(q, 0, 7, 10000.0, np.zeros((0, d)), k[None, :])
    s = O.rope(q, 7, 10000.0) @ O.rope(k, 7, 10000.0) / math.sqrt(d)
    assert abs(lse - s) < 1e-12


def test_identical_keys_add_log_n():
    rng = np.random.default_rng(1)
    d, n = 64, 13
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    mem = np.repeat(k[None, :], n, axis=0)
    lse = O.routed_attention_row_lse(q, 0, 0, 10000.0, mem, np.zeros((1, d)))   # plus local key 0 = 0: logit 0
    s = O.rope(q, 0, 10000.0) @ k / math.sqrt(d)
    assert abs(lse - math.log(n * math.exp(s) + 1.0)) < 1e-12


def test_normalises_the_row_softmax():
    rng = np.random.default_rng(2)
    q, qi, koff, base, mk, mv, lk, lv = _row(rng)
    lse = O.routed_attention_row_lse(q, qi, koff, base, mk, lk)
    q_rot = O.rope(q, koff + qi, base)
    keys = np.concatenate([mk, O.rope(lk[:qi + 1], koff + np.arange(qi + 1), base)])
    vals = np.concatenate([mv, lv[:qi + 1]])
    w = np.exp(keys @ q_rot / math.sqrt(q.shape[0]) - lse)
    assert abs(w.sum() - 1.0) < 1e-12
    np.testing.assert_allclose(w @ vals, O.routed_attention_row(q, qi, koff, base, mk, mv, lk, lv), atol=1e-12)


def test_key_order_invariant():
    rng = np.random.default_rng(3)
    q, qi, koff, base, mk, mv, lk, lv = _row(rng)
    a = O.routed_attention_row_lse(q, qi, koff, base, mk, lk)
    b = O.routed_attention_row_lse(q, qi, koff, base, mk[::-1], lk)
    assert abs(a - b) < 1e-12


def test_planted_log2_fails():
    rng = np.random.default_rng(4)
    q, qi, koff, base, mk, mv, lk, lv = _row(rng)
    lse = O.routed_attention_row_lse(q, qi, koff, base, mk, lk)
    q_rot = O.rope(q, koff + qi, base)
    keys = np.concatenate([mk, O.rope(lk[:qi + 1], koff + np.arange(qi + 1), base)])
    s = keys @ q_rot / math.sqrt(q.shape[0])
    wrong = s.max() + math.log2(np.exp(s - s.max()).sum())
    assert abs(np.exp(s - wrong).sum() - 1.0) > 1e-3
    assert abs(lse - wrong) > 1e-3
