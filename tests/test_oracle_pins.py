"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an invariant, an independent formulation, a library routine in a
special case, or brute force on tiny inputs. Citations name the page and the
section the checked fact comes from.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import msa_oracle as O

rng = np.random.default_rng(1234)


# ---------------------------------------------------------------- pooling
# "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术" §2.1 item 2, §3.1: 256-token chunk means.

RAGGED_LENS = [1, 255, 256, 257, 511, 513, 700]


def test_pool_ramp_midpoints_ragged():
    """R[t] = (t+1) e within a document: each chunk's mean is the midpoint of its
    actual token range, (s + e + 1) / 2, including the ragged last chunk."""
    d = 8
    for L in RAGGED_LENS:
        R = np.outer(np.arange(1, L + 1, dtype=np.float64), np.ones(d))
        kr = O.chunk_mean_pool(R)
        assert kr.shape == (math.ceil(L / 256), d)
        for c in range(kr.shape[0]):
            s, e = 256 * c, min(256 * (c + 1), L)
            np.testing.assert_allclose(kr[c], (s + e + 1) / 2.0, rtol=0, atol=1e-12)


def test_pool_bank_owner_and_boundaries():
    """Chunks never cross documents: doc j's chunks see only doc j's ramp values."""
    d = 4
    lens = RAGGED_LENS
    off = O.doc_offsets(lens)
    R = np.zeros((int(off[-1]), d))
    for j, L in enumerate(lens):
        R[off[j]:off[j + 1]] = (1000.0 * j + np.arange(L))[:, None]
    kr, owner = O.build_routing_keys(R, lens)
    assert kr.shape[0] == sum(math.ceil(L / 256) for L in lens)
    c = 0
    for j, L in enumerate(lens):
        for s in range(0, L, 256):
            e = min(s + 256, L)
            assert owner[c] == j
            np.testing.assert_allclose(kr[c], 1000.0 * j + (s + e - 1) / 2.0, atol=1e-9)
            c += 1


def test_pool_divisible_equals_page_view_mean():
    """For lengths divisible by 256 the page's example (view into
    [.., L/256, 256, d] then mean over the chunk axis) gives the same K_r."""
    d = 16
    for L in (256, 512, 1024):
        x = torch.from_numpy(rng.standard_normal((1, L, d)))
        page = x.view(-1, L // 256, 256, d).mean(dim=2)[0].numpy()
        np.testing.assert_allclose(O.chunk_mean_pool(x[0].numpy()), page, rtol=1e-12, atol=1e-12)


def test_pool_constant():
    R = np.full((300, 5), -2.5)
    np.testing.assert_array_equal(O.chunk_mean_pool(R), np.full((2, 5), -2.5))


def test_doc_offsets_reject_empty_doc():
    with pytest.raises(ValueError):
        O.doc_offsets([3, 0, 2])


# ---------------------------------------------------------------- RoPE
# "MSA架构…" §2.2 and robocikowo.com "Komponenty": document-wise (Parallel) RoPE,
# Global RoPE with a k-offset for the active context.

def test_rope_equals_complex_rotation():
    """Independent formulation: (x_i + j x_{i+d/2}) * exp(j p theta_i)."""
    for d, base in ((8, 10000.0), (64, 10000.0), (128, 500.0)):
        x = rng.standard_normal((5, d))
        pos = np.array([0, 1, 7, 4095, 524287])
        z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(
            1j * pos[:, None] * (base ** (-np.arange(0, d, 2) / d))[None, :])
        ref = np.concatenate([z.real, z.imag], axis=1)
        np.testing.assert_allclose(O.rope(x, pos, base), ref, rtol=1e-9, atol=1e-9)


def test_rope_hand_values_d4():
    """Hand-derived, d = 4, base 10000: theta = (1, 1/100); x = (1, 2, 3, 4) at
    position 3 turns pair (x0, x2) by 3 rad and pair (x1, x3) by 0.03 rad."""
    c, s, c2, s2 = math.cos(3), math.sin(3), math.cos(0.03), math.sin(0.03)
    expected = [1 * c - 3 * s, 2 * c2 - 4 * s2, 3 * c + 1 * s, 4 * c2 + 2 * s2]
    np.testing.assert_allclose(O.rope(np.array([1.0, 2, 3, 4]), 3, 10000.0), expected,
                               rtol=0, atol=1e-14)


def test_rope_invariants():
    d = 64
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    np.testing.assert_array_equal(O.rope(q, 0, 10000.0), q)          # position 0: unchanged
    r = O.rope(q, 1234, 10000.0)
    np.testing.assert_allclose(r[:32] ** 2 + r[32:] ** 2, q[:32] ** 2 + q[32:] ** 2, rtol=1e-12)
    for p, pp, delta in ((5, 3, 100), (1000, 4000, 65536), (0, 70000, 17)):
        a = O.rope(q, p, 10000.0) @ O.rope(k, pp, 10000.0)
        b = O.rope(q, p + delta, 10000.0) @ O.rope(k, pp + delta, 10000.0)
        assert abs(a - b) < 1e-9                                      # relative positions only
    # sign: turning by +p then by -p returns the vector
    np.testing.assert_allclose(O.rope(O.rope(q, 77, 10000.0), -77, 10000.0), q, atol=1e-12)


def test_parallel_rope_resets_per_document():
    lens = [3, 5, 2]
    d = 8
    K = rng.standard_normal((10, d))
    out = O.parallel_rope_bank(K, lens, 10000.0)
    expected_pos = [0, 1, 2, 0, 1, 2, 3, 4, 0, 1]
    for t, p in enumerate(expected_pos):
        z = (K[t, :4] + 1j * K[t, 4:]) * np.exp(1j * p * 10000.0 ** (-np.arange(0, d, 2) / d))
        np.testing.assert_allclose(out[t], np.concatenate([z.real, z.imag]), atol=1e-12)


def test_k_offset():
    assert O.k_offset(2, [512] * 16) == 1024
    assert O.k_offset(32, [600, 16383, 513]) == 32 * 16383


# ---------------------------------------------------------------- routing
# "MSA架构…" §2.1 item 1: cosine-similarity top-k router; robocikowo.com "Komponenty".

def _toy_bank(lens, d=16):
    off = O.doc_offsets(lens)
    R = rng.standard_normal((int(off[-1]), d))
    kr, owner = O.build_routing_keys(R, lens)
    return R, kr, owner


@pytest.mark.parametrize("vectorised", [False, True])
def test_router_self_match_scores_one(vectorised):
    lens = [300, 256, 600, 10]
    _, kr, owner = _toy_bank(lens)
    for c in range(kr.shape[0]):
        if vectorised:
            s = O.doc_max(O.chunk_cosines(kr[c], kr), owner, len(lens))
        else:
            s = O.route_doc_scores(kr[c], kr, owner, len(lens))
        assert abs(s[owner[c]] - 1.0) < 1e-12
        assert np.all(s <= 1.0 + 1e-12) and np.all(s >= -1.0 - 1e-12)


@pytest.mark.parametrize("vectorised", [False, True])
def test_router_max_over_chunks_not_mean(vectorised):
    """Doc 0 has 3 chunks; q matches only its middle chunk -> score 1, while
    the cosine against the document's mean key would be well below 1."""
    d = 16
    lens = [700, 256]
    R = rng.standard_normal((956, d))
    kr, owner = O.build_routing_keys(R, lens)
    q = kr[1] * 3.0
    s = (O.doc_max(O.chunk_cosines(q, kr), owner, 2) if vectorised
         else O.route_doc_scores(q, kr, owner, 2))
    assert abs(s[0] - 1.0) < 1e-12
    assert O.cosine(q, R[:700].mean(axis=0)) < 0.9
    # anti-aligned single-chunk document scores -1
    s2 = O.route_doc_scores(-kr[3], kr, owner, 2)
    assert abs(s2[1] + 1.0) < 1e-12


def test_router_scale_invariance_and_brute_force():
    lens = [257, 1000, 31]
    _, kr, owner = _toy_bank(lens)
    q = rng.standard_normal(16)
    s1 = O.route_doc_scores(q, kr, owner, 3)
    s7 = O.route_doc_scores(7.0 * q, kr, owner, 3)
    np.testing.assert_allclose(s1, s7, atol=1e-14)
    for j in range(3):                               # brute force: angle between vectors
        cs = [np.cos(np.arccos(np.clip(q @ kr[c] / np.linalg.norm(q) / np.linalg.norm(kr[c]),
                                       -1, 1))) for c in range(kr.shape[0]) if owner[c] == j]
        assert abs(s1[j] - max(cs)) < 1e-12
    np.testing.assert_allclose(O.doc_max(O.chunk_cosines(q, kr), owner, 3), s1, atol=1e-14)


def test_router_zero_vector_scores_zero():
    assert O.cosine(np.zeros(4), np.ones(4)) == 0.0


def test_block_mean_query():
    Qr = np.arange(8 * 3, dtype=np.float64).reshape(8, 3)
    got = O.block_mean_query(Qr, 4)
    np.testing.assert_allclose(got, [Qr[:4].sum(0) / 4, Qr[4:].sum(0) / 4])
    np.testing.assert_array_equal(O.block_mean_query(Qr, 1), Qr)
    with pytest.raises(ValueError):
        O.block_mean_query(Qr, 3)


# ---------------------------------------------------------------- top-k
# robocikowo.com "Hiperparametry" (Top-k documents) and "Paradygmat wykonania".

def _brute_top_k(s, k):
    """The unique k-subset whose members all beat all non-members under
    (score desc, index asc), found by enumerating every subset."""
    n = len(s)
    beats = lambda a, b: s[a] > s[b] or (s[a] == s[b] and a < b)
    for sub in itertools.combinations(range(n), k):
        rest = [b for b in range(n) if b not in sub]
        if all(beats(a, b) for a in sub for b in rest):
            return set(sub)
    raise AssertionError("no dominating subset")


def test_top_k_brute_force_with_ties():
    for trial in range(200):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, n + 1))
        s = rng.integers(-3, 4, size=n).astype(np.float64) / 3.0     # many ties
        got = O.select_top_k(s, k)
        assert set(got.tolist()) == _brute_top_k(s, k)
        for a, b in zip(got[:-1], got[1:]):                          # output order
            assert s[a] > s[b] or (s[a] == s[b] and a < b)


def test_top_k_permutation():
    s = rng.standard_normal(50)
    perm = rng.permutation(50)
    got = O.select_top_k(s, 7)
    got_p = O.select_top_k(s[perm], 7)
    np.testing.assert_array_equal(perm[got_p], got)
    with pytest.raises(ValueError):
        O.select_top_k(s, 51)


# ---------------------------------------------------------------- attention
# robocikowo.com "Komponenty" (append the selected documents' K/V to the local
# context; Global RoPE), "Paradygmat wykonania" (only the k selected take part).

def _small_inputs(B=1, Hq=4, Hkv=2, d=16, lens=(40, 70, 25, 64), Lc=12, Tq=4, seed=0):
    r = np.random.default_rng(seed)
    N = int(sum(lens))
    return {
        "K": r.standard_normal((Hkv, N, d)), "V": r.standard_normal((Hkv, N, d)),
        "R": r.standard_normal((Hkv, N, d)), "Q": r.standard_normal((B, Hq, Tq, d)),
        "Qr": r.standard_normal((B, Hkv, Tq, d)), "LK": r.standard_normal((B, Hkv, Lc, d)),
        "LV": r.standard_normal((B, Hkv, Lc, d)),
    }, list(lens)


def test_attention_rows_sum_to_one():
    inp, lens = _small_inputs()
    inp["V"][:] = 1.0
    inp["LV"][:] = 1.0
    out = O.forward(inp, lens, top_k=2, route_block=2)["out"]
    np.testing.assert_allclose(out, 1.0, atol=1e-12)


def test_attention_zero_query_is_mean_of_visible_values():
    inp, lens = _small_inputs()
    inp["Q"][:] = 0.0
    res = O.forward(inp, lens, top_k=2, route_block=4)
    off = O.doc_offsets(lens)
    Lc, Tq, G = 12, 4, 2
    for hq in range(4):
        h = hq // G
        docs = res["topk"][0, 0, h]
        mem = np.concatenate([inp["V"][h, off[j]:off[j + 1]] for j in docs])
        for t in range(Tq):
            i = Lc - Tq + t
            vis = np.concatenate([mem, inp["LV"][0, h, :i + 1]])
            np.testing.assert_allclose(res["out"][0, hq, t], vis.mean(axis=0), atol=1e-12)


def _dense_reference(inp, lens, k_off, base=10000.0):
    """Every document selected: one SDPA call (fp64) over the whole bank plus the
    causal local context, positions written out here independently."""
    K, V, Q, LK, LV = (torch.from_numpy(inp[x]) for x in ("K", "V", "Q", "LK", "LV"))
    Hkv, N, d = K.shape
    B, Hq, Tq, _ = Q.shape
    Lc = LK.shape[2]
    G = Hq // Hkv
    inv = base ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)

    def turn(x, pos):
        z = torch.complex(x[..., : d // 2], x[..., d // 2:]) * torch.polar(
            torch.ones_like(pos[..., None] * inv), pos[..., None] * inv)
        return torch.cat([z.real, z.imag], dim=-1)

    doc_pos = torch.cat([torch.arange(L, dtype=torch.float64) for L in lens])
    loc_pos = k_off + torch.arange(Lc, dtype=torch.float64)
    keys = torch.cat([turn(K, doc_pos).unsqueeze(0).expand(B, -1, -1, -1), turn(LK, loc_pos)], 2)
    vals = torch.cat([V.unsqueeze(0).expand(B, -1, -1, -1), LV], 2)
    keys = keys.repeat_interleave(G, dim=1)
    vals = vals.repeat_interleave(G, dim=1)
    qi = Lc - Tq + torch.arange(Tq)
    q = turn(Q, (k_off + qi).to(torch.float64))
    mask = torch.cat([torch.ones(Tq, N, dtype=torch.bool),
                      torch.arange(Lc)[None, :] <= qi[:, None]], dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, keys, vals, attn_mask=mask).numpy()


def test_all_documents_selected_equals_dense_sdpa():
    inp, lens = _small_inputs(B=2, Hq=6, Hkv=3, d=16, lens=(40, 70, 25, 64, 9), Lc=10, Tq=6)
    n = len(lens)
    res = O.forward(inp, lens, top_k=n, route_block=3)
    assert res["k_off"] == n * max(lens)
    ref = _dense_reference(inp, lens, res["k_off"])
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


def test_bank_permutation_invariance():
    inp, lens = _small_inputs(lens=(33, 80, 51, 64, 20))
    base = O.forward(inp, lens, top_k=3, route_block=4)
    perm = [3, 0, 4, 2, 1]
    off = O.doc_offsets(lens)
    inp2 = dict(inp)
    for name in ("K", "V", "R"):
        inp2[name] = np.concatenate([inp[name][:, off[j]:off[j + 1]] for j in perm], axis=1)
    lens2 = [lens[j] for j in perm]
    res = O.forward(inp2, lens2, top_k=3, route_block=4)
    np.testing.assert_array_equal(np.asarray(perm)[res["topk"]], base["topk"])
    np.testing.assert_allclose(res["out"], base["out"], rtol=1e-12, atol=1e-13)


def test_single_token_document_and_single_local_token():
    """One document of one token, Lc = Tq = 1: a two-key softmax by hand.
    k_off = 1 * 1, the memory key sits at position 0, the local key and the
    query at position 1 (same position: the local logit is the plain dot)."""
    d = 8
    r = np.random.default_rng(5)
    q, km, vm, kl, vl = (r.standard_normal(d) for _ in range(5))
    inp = {"K": km.reshape(1, 1, d), "V": vm.reshape(1, 1, d), "R": r.standard_normal((1, 1, d)),
           "Q": q.reshape(1, 1, 1, d), "Qr": r.standard_normal((1, 1, 1, d)),
           "LK": kl.reshape(1, 1, 1, d), "LV": vl.reshape(1, 1, 1, d)}
    out = O.forward(inp, [1], top_k=1, route_block=1)["out"][0, 0, 0]
    z = (q[:4] + 1j * q[4:]) * np.exp(1j * 10000.0 ** (-np.arange(0, d, 2) / d))
    a = np.concatenate([z.real, z.imag]) @ km / math.sqrt(d)
    b = q @ kl / math.sqrt(d)
    np.testing.assert_allclose(out, (math.exp(a) * vm + math.exp(b) * vl) / (math.exp(a) + math.exp(b)),
                               atol=1e-12)


def test_causality_of_local_context():
    inp, lens = _small_inputs(Lc=12, Tq=4)
    base = O.forward(inp, lens, top_k=2, route_block=4)["out"]
    inp2 = {k: v.copy() for k, v in inp.items()}
    inp2["LK"][:, :, 10:] += 5.0       # local tokens 10, 11: queries 8, 9 cannot see them
    inp2["LV"][:, :, 10:] -= 3.0
    out2 = O.forward(inp2, lens, top_k=2, route_block=4)["out"]
    np.testing.assert_array_equal(out2[:, :, :2], base[:, :, :2])    # queries at 8, 9
    assert np.abs(out2[:, :, 2:] - base[:, :, 2:]).max() > 1e-3      # 10, 11 see them


def test_gqa_head_mapping():
    inp, lens = _small_inputs(Hq=6, Hkv=3)
    for h in range(3):
        inp["V"][h] = h + 1.0
        inp["LV"][:, h] = h + 1.0
    out = O.forward(inp, lens, top_k=2, route_block=2)["out"]
    for hq in range(6):
        np.testing.assert_allclose(out[:, hq], hq // 2 + 1.0, atol=1e-12)


def test_selection_override_and_oracle_topk_consistent():
    inp, lens = _small_inputs()
    res = O.forward(inp, lens, top_k=2, route_block=4)
    again = O.forward(inp, lens, top_k=2, route_block=4, selection=res["topk"])
    np.testing.assert_array_equal(again["out"], res["out"])
    # the chosen documents are the two best by routing score
    for h in range(2):
        s = res["doc_scores"][0, 0, h]
        assert set(res["topk"][0, 0, h]) == set(np.argsort(-s, kind="stable")[:2])


def test_oracle_regression_fixture():
    """The oracle still reproduces tests/golden/tiny_forward.json (make_golden.py)."""
    import json
    from tests.golden import make_golden as MG
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_forward.json")) as f:
        g = json.load(f)
    res = O.forward(MG.inputs(g["spec"]), g["spec"]["lens"], g["spec"]["top_k"],
                    g["spec"]["route_block"])
    np.testing.assert_array_equal(res["topk"], g["topk"])
    np.testing.assert_allclose(res["out"], g["out"], atol=1e-11)
    np.testing.assert_allclose(res["doc_scores"], g["doc_scores"], atol=1e-11)
