"""Pins of the oracle's Memory Interleave (CPU only).

One hop is the routed step itself; hops never re-select a document; when the hops
have taken every document, the last attention is dense attention over the whole
bank (an independent formulation); a document's routing key is the token mean,
which equals the chunk means weighted by chunk length; the next query follows the
stated update in closed form on orthonormal keys; and a planted two-hop chain is
found only because of the update (a bridge document, then the document that is
near the bridge but not near the query). Planted mistakes fail these pins."""
import math

import numpy as np
import pytest

from oracle import msa_oracle as O
from tests.test_oracle_pins import _dense_reference


def _inputs(seed, Hkv, G, d, lens, B, Tq, Lc):
    rng = np.random.default_rng(seed)
    N = int(sum(lens))
    return {"K": rng.standard_normal((Hkv, N, d)), "V": rng.standard_normal((Hkv, N, d)),
            "R": rng.standard_normal((Hkv, N, d)), "Q": rng.standard_normal((B, Hkv * G, Tq, d)),
            "Qr": rng.standard_normal((B, Hkv, Tq, d)), "LK": rng.standard_normal((B, Hkv, Lc, d)),
            "LV": rng.standard_normal((B, Hkv, Lc, d))}


LENS = [300, 5, 257, 1, 40, 513, 90, 256, 7, 120, 33, 600]


def test_one_hop_is_the_routed_step():
    inp = _inputs(1, 2, 2, 8, LENS, 2, 4, 9)
    ref = O.forward(inp, LENS, 3, 2)
    res = O.memory_interleave(inp, LENS, 3, 2, hops=1)
    np.testing.assert_array_equal(res["topk"][0], ref["topk"])
    np.testing.assert_allclose(res["out"][0], ref["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["q_r"][0], ref["q_r"], rtol=0, atol=1e-12)


def test_hops_take_new_documents_and_all_documents_give_dense_attention():
    inp = _inputs(2, 2, 2, 8, LENS, 2, 2, 5)
    k, hops = 3, 4                                      # 4 hops x 3 = all 12 documents
    res = O.memory_interleave(inp, LENS, k, 1, hops=hops)
    for t in range(hops):
        sel = res["selection"][t]
        assert sel.shape[-1] == (t + 1) * k
        for row in sel.reshape(-1, sel.shape[-1]):
            assert len(set(row.tolist())) == len(row)      # no document twice
        np.testing.assert_array_equal(sel[..., t * k:], res["topk"][t])
    dense = _dense_reference(inp, LENS, O.k_offset(len(LENS), LENS), 10000.0)
    np.testing.assert_allclose(res["out"][-1], dense, rtol=0, atol=1e-12)


def test_doc_routing_key_is_the_length_weighted_chunk_mean():
    rng = np.random.default_rng(3)
    for L in (1, 255, 256, 257, 700):
        R = rng.standard_normal((L, 6))
        kr = O.chunk_mean_pool(R)
        w = np.array([e - s for s, e in O.chunk_spans(L)], dtype=np.float64)
        np.testing.assert_allclose(O.doc_routing_key(R), (w @ kr) / L, rtol=0, atol=1e-12)
        np.testing.assert_allclose(O.doc_routing_key(R), R.mean(axis=0), rtol=0, atol=1e-12)


def test_next_query_closed_form():
    e = np.eye(6)
    q = 3.0 * e[0]                                   # |q| = 3
    nxt = O.interleave_next_query(q, [2.0 * e[1], 5.0 * e[4]])
    np.testing.assert_allclose(nxt, e[0] + 0.5 * e[1] + 0.5 * e[4], rtol=0, atol=1e-15)


def _chain_bank():
    """Five one-token documents in d = 8 (K_r of a one-token document is that token):
    A = (e0 + e1)/sqrt2 (the bridge), B = e1 (the target), C = -e0,
    D = (0.1 e0 + e2) normalised (a distractor slightly nearer the query than B), E = e3.
    The query routes with q = e0 and top_k = 1."""
    e = np.eye(8)
    keys = [(e[0] + e[1]) / math.sqrt(2), e[1], -e[0], (0.1 * e[0] + e[2]) / np.linalg.norm(0.1 * e[0] + e[2]), e[3]]
    lens = [1] * 5
    rng = np.random.default_rng(4)
    inp = {"K": rng.standard_normal((1, 5, 8)), "V": rng.standard_normal((1, 5, 8)),
           "R": np.stack(keys)[None], "Q": rng.standard_normal((1, 1, 1, 8)), "Qr": e[0][None, None, None],
           "LK": rng.standard_normal((1, 1, 2, 8)), "LV": rng.standard_normal((1, 1, 2, 8))}
    return inp, lens


def test_planted_chain_needs_the_update():
    inp, lens = _chain_bank()
    res = O.memory_interleave(inp, lens, 1, 1, hops=2)
    assert res["topk"][0][0, 0, 0, 0] == 0             # the bridge
    assert res["topk"][1][0, 0, 0, 0] == 1             # then the target, through the bridge's key
    # without the update the second hop picks the distractor: the pin sees the update
    good = O.interleave_next_query
    try:
        O.interleave_next_query = lambda q, keys: np.asarray(q, dtype=np.float64)
        assert O.memory_interleave(inp, lens, 1, 1, hops=2)["topk"][1][0, 0, 0, 0] == 3
    finally:
        O.interleave_next_query = good


def test_planted_mistake_reselection_fails():
    inp = _inputs(5, 1, 2, 8, LENS, 1, 1, 3)
    good = O.select_top_k_excluding
    try:
        O.select_top_k_excluding = lambda s, k, ex: O.select_top_k(s, k)   # forgets the context
        res = O.memory_interleave(inp, LENS, 2, 1, hops=3)
        rows = res["selection"][-1].reshape(-1, 6)
        assert any(len(set(r.tolist())) < 6 for r in rows)
    finally:
        O.select_top_k_excluding = good
    with pytest.raises(ValueError):
        O.select_top_k_excluding(np.zeros(4), 3, [0, 1])
