"""Pins of the oracle's reduced-precision router variant (normalised routing keys
stored in bf16): the bf16 rounding itself against values the format fixes, exact
agreement with the cosine where the normalised keys are bf16 numbers, the rounding
bound elsewhere, and a planted mistake (rounding the query instead) failing."""
import math

import numpy as np

from oracle import msa_oracle as O


def test_round_bf16_fixed_values():
    r = O.round_bf16
    assert r(1.0) == 1.0
    assert r(1.0 + 2.0 ** -8) == 1.0                       # halfway, to the even mantissa
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6       # halfway, to the even mantissa (up)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7  # past halfway: up
    assert r(-3.0) == -3.0
    assert r(math.pi) == 3.140625                           # 8 significant bits of pi
    assert r(0.1) == 0.10009765625
    assert r(0.0) == 0.0
    x = np.random.default_rng(0).standard_normal(1000)
    rel = np.abs(r(x) - x) / np.abs(x)
    assert rel.max() <= 2.0 ** -8                           # unit roundoff of 8 significant bits


def _keys_exact_in_bf16(rng, n, d):
    """Unit keys with four +-1/2 components: k / |k| = k is a bf16 vector."""
    K = np.zeros((n, d))
    for c in range(n):
        idx = rng.choice(d, size=4, replace=False)
        K[c, idx] = rng.choice([-0.5, 0.5], size=4)
    return K * rng.uniform(0.5, 3.0, size=(n, 1))           # any positive scale: the cosine undoes it


def test_bf16_keys_equal_the_cosine_when_keys_are_bf16():
    rng = np.random.default_rng(1)
    K = _keys_exact_in_bf16(rng, 40, 128)
    q = rng.standard_normal(128)
    exact = np.array([O.cosine(q, k) for k in K])
    np.testing.assert_allclose(O.chunk_cosines_bf16_keys(q, K), exact, rtol=0, atol=1e-15)


def test_bf16_keys_rounding_bound():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((300, 128))
    q = rng.standard_normal(128)
    exact = np.array([O.cosine(q, k) for k in K])
    got = O.chunk_cosines_bf16_keys(q, K)
    qh = q / np.linalg.norm(q)
    kh = K / np.linalg.norm(K, axis=1, keepdims=True)
    bound = 2.0 ** -8 * np.abs(kh * qh).sum(axis=1)
    assert np.all(np.abs(got - exact) <= bound + 1e-15)
    assert np.abs(got - exact).max() > 0                    # the variant is not the exact cosine


def test_planted_query_rounding_fails_the_exact_case():
    rng = np.random.default_rng(3)
    K = _keys_exact_in_bf16(rng, 40, 128)
    q = rng.standard_normal(128)

    def wrong(q_r, K_r):                                     # rounds q^ instead of k^
        qh = O.round_bf16(q_r / np.linalg.norm(q_r))
        return (K_r / np.linalg.norm(K_r, axis=1, keepdims=True)) @ qh

    exact = np.array([O.cosine(q, k) for k in K])
    assert np.abs(wrong(q, K) - exact).max() > 1e-6


def test_forward_router_keys_option():
    rng = np.random.default_rng(4)
    lens = [300, 260, 40]
    H, d = 1, 64
    N = sum(lens)
    inp = {"K": rng.standard_normal((H, N, d)), "V": rng.standard_normal((H, N, d)),
           "R": rng.standard_normal((H, N, d)), "Q": rng.standard_normal((1, 2, 2, d)),
           "Qr": rng.standard_normal((1, H, 2, d)), "LK": rng.standard_normal((1, H, 4, d)),
           "LV": rng.standard_normal((1, H, 4, d))}
    a = O.forward(inp, lens, 2, 1)
    b = O.forward(inp, lens, 2, 1, router_keys="bf16")
    diff = np.abs(a["doc_scores"] - b["doc_scores"])
    assert diff.max() <= 2.0 ** -8 and diff.max() > 0
