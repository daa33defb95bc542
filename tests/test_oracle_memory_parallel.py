"""Pins of the oracle's Memory Parallel functions (CPU only).

The sharded step is the same definition as the single-bank step, so the pins are
identities the mathematics fixes: the merge of the shards' local top-k lists is the
global top-k of all scores (brute-force sort), the merge of partial softmaxes over
disjoint key subsets is the softmax over their union (closed form), and the whole
sharded step equals forward() for every shard count. Planted mistakes in the merge
rules (placed in the oracle module for the test, on the CPU) fail them."""
import math

import numpy as np
import pytest

from oracle import msa_oracle as O


def test_shard_ranges_cover_contiguously():
    for n in (1, 2, 7, 16, 33):
        for s in range(1, min(n, 6) + 1):
            r = O.shard_ranges(n, s)
            assert r[0][0] == 0 and r[-1][1] == n and len(r) == s
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [hi - lo for lo, hi in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        O.shard_ranges(3, 4)


def test_merge_candidates_is_the_global_top_k():
    rng = np.random.default_rng(0)
    for trial in range(200):
        n = int(rng.integers(2, 40))
        k = int(rng.integers(1, n + 1))
        # few distinct values: exact ties inside and across shards
        scores = rng.integers(-3, 4, n).astype(np.float64) / 4.0
        S = int(rng.integers(1, min(n, 6) + 1))
        cs, ci = [], []
        for lo, hi in O.shard_ranges(n, S):
            loc = O.select_top_k(scores[lo:hi], min(k, hi - lo))
            ci.append(loc + lo)
            cs.append(scores[lo:hi][loc])
        idx, sc = O.merge_candidates(cs, ci, k)
        brute = sorted(range(n), key=lambda j: (-scores[j], j))[:k]
        np.testing.assert_array_equal(idx, brute)
        np.testing.assert_array_equal(sc, scores[brute])


def _rand_row(rng, m, d):
    q = rng.standard_normal(d)
    return q, rng.standard_normal((m, d)) * 2.0, rng.standard_normal((m, d))


def test_merge_partials_is_the_softmax_over_the_union():
    rng = np.random.default_rng(1)
    for trial in range(100):
        d, m = int(rng.choice([4, 16, 64])), int(rng.integers(1, 300))
        q, K, V = _rand_row(rng, m, d)
        whole = O.softmax_attention(q, K, V)
        s = K @ q / math.sqrt(d)
        lse_all = s.max() + math.log(np.exp(s - s.max()).sum())
        parts = int(rng.integers(1, 6))
        cut = np.sort(rng.integers(0, m + 1, parts - 1))
        bounds = [0, *cut.tolist(), m]              # may hold empty parts
        outs, lses = zip(*[O.attention_partial(q, K[a:b], V[a:b]) for a, b in zip(bounds, bounds[1:])])
        out, L = O.merge_partials(outs, lses)
        np.testing.assert_allclose(out, whole, rtol=0, atol=1e-12)
        assert abs(L - lse_all) <= 1e-12


def test_empty_partials():
    out, lse = O.attention_partial(np.ones(8), np.zeros((0, 8)), np.zeros((0, 8)))
    assert lse == -math.inf and not out.any()
    out, L = O.merge_partials([np.ones(8), np.ones(8)], [-math.inf, -math.inf])
    assert L == -math.inf and not out.any()


def _inputs(seed, Hkv, G, d, lens, B, Tq, Lc):
    rng = np.random.default_rng(seed)
    N = int(sum(lens))
    return {"K": rng.standard_normal((Hkv, N, d)), "V": rng.standard_normal((Hkv, N, d)),
            "R": rng.standard_normal((Hkv, N, d)), "Q": rng.standard_normal((B, Hkv * G, Tq, d)),
            "Qr": rng.standard_normal((B, Hkv, Tq, d)), "LK": rng.standard_normal((B, Hkv, Lc, d)),
            "LV": rng.standard_normal((B, Hkv, Lc, d))}


CASE = dict(seed=3, Hkv=2, G=2, d=8, lens=[300, 5, 257, 1, 40, 513, 90, 256, 7, 120], B=2, Tq=4, Lc=9)


@pytest.mark.parametrize("n_shards,owner", [(1, 0), (2, 0), (3, 2), (5, 1), (10, 4)])
def test_sharded_step_equals_the_single_bank_step(n_shards, owner):
    c = CASE
    inp = _inputs(c["seed"], c["Hkv"], c["G"], c["d"], c["lens"], c["B"], c["Tq"], c["Lc"])
    k, Bq = 3, 2
    ref = O.forward(inp, c["lens"], k, Bq)
    mp = O.memory_parallel_forward(inp, c["lens"], k, Bq, n_shards, owner=owner)
    np.testing.assert_array_equal(mp["topk"], ref["topk"])
    np.testing.assert_allclose(mp["out"], ref["out"], rtol=0, atol=1e-12)
    # only the owner attends the local context; the partial of a shard holding none of
    # a row's documents and not the owner is empty
    assert np.isfinite(mp["part_lse"][owner]).all()


def test_planted_merge_mistakes_fail():
    c = CASE
    inp = _inputs(c["seed"], c["Hkv"], c["G"], c["d"], c["lens"], c["B"], c["Tq"], c["Lc"])
    ref = O.forward(inp, c["lens"], 3, 2)
    good_p, good_c = O.merge_partials, O.merge_candidates

    def max_weighted(outs, lses):  # weights exp(lse - max) without renormalising
        m = max(x for x in lses if x != -math.inf)
        return sum(math.exp(x - m) * np.asarray(o) for o, x in zip(outs, lses) if x != -math.inf), m

    def ties_high(cs, ci, k):      # equal scores to the higher index
        pairs = sorted(((-float(s), -int(j)) for a, b in zip(cs, ci) for s, j in zip(a, b)))[:k]
        return np.asarray([-j for _, j in pairs]), np.asarray([-s for s, _ in pairs])

    try:
        O.merge_partials = max_weighted
        mp = O.memory_parallel_forward(inp, c["lens"], 3, 2, 3)
        assert np.abs(mp["out"] - ref["out"]).max() > 1e-3
    finally:
        O.merge_partials = good_p
    # a tie-order mistake shows on exactly tied candidates
    cs, ci = [np.array([0.5, 0.25])], [np.array([4, 9])]
    cs.append(np.array([0.5, 0.1]))
    ci.append(np.array([2, 7]))
    assert list(good_c(cs, ci, 2)[0]) == [2, 4]
    assert list(ties_high(cs, ci, 2)[0]) != [2, 4]
