"""Memory Interleave through the C ABI (msa_interleave_route + msa_attend per hop)
against the oracle, hop by hop.

Each hop is checked given the GPU's own earlier hops (so a near tie in one hop does
not carry into the next comparison): the hop's routing query against the oracle's
update of the previous query by the previous hop's documents; the hop's new
documents against the oracle's top-k over the documents outside the context (exact
set, or differing only inside the near-tie window), their scores within 1e-3; the
context has no document twice; the attention over the expanded context against
the oracle over the same selection. When the hops take every document, the last
attention is dense attention over the bank."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "decode": (Workload("il_decode", 51, 2, 8, 2, 128, 40, 0, 200, 1, 1, 4, ragged=(1, 900)), 3),
    "blocks": (Workload("il_blocks", 52, 1, 4, 2, 64, 30, 0, 96, 8, 4, 3, ragged=(50, 600)), 4),
    "f32": (Workload("il_f32", 53, 2, 4, 2, 128, 24, 0, 64, 1, 1, 3, ragged=(1, 500), dtype="f32"), 3),
    # 5 hops x 4 = every document: the last hop is dense attention over the bank
    "all_docs": (Workload("il_all", 54, 1, 4, 1, 64, 20, 0, 48, 2, 2, 4, ragged=(1, 200)), 5),
}


def _run(w, hops):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    sh = torch.cuda.current_stream().cuda_stream
    nblk = w.q_tokens // w.route_block
    B, Hkv, d, k = w.batch, w.n_kv_heads, w.head_dim, w.top_k
    q_in, ctx, hops_out = None, None, []
    for t in range(hops):
        ctx_out = torch.full((B, nblk, Hkv, (t + 1) * k), -7, dtype=torch.int32, device="cuda")
        tsc = torch.empty((B, nblk, Hkv, k), dtype=torch.float32, device="cuda")
        q_out = torch.empty((B, Hkv, nblk, d), dtype=torch.float32, device="cuda")
        msa.msa_interleave_route(bank.handle, qry, k, 0 if q_in is None else q_in.data_ptr(),
                                 0 if ctx is None else ctx.data_ptr(), t * k, ctx_out.data_ptr(), tsc.data_ptr(),
                                 q_out.data_ptr(), sh)
        out = bank.attend(qry, (t + 1) * k, ctx_out)
        hops_out.append({"ctx": ctx_out, "tsc": tsc, "q_out": q_out, "out": out})
        ctx, q_in = ctx_out, q_out
    # the Python hop loop runs the same calls
    from sparse_attention_routed_b200.interleave import run_hops
    loop = run_hops(bank, qry, k, hops)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    for h, (c2, o2) in zip(hops_out, loop):
        assert torch.equal(h["ctx"], c2) and torch.equal(h["out"], o2)
    res = [{kk: v.cpu().numpy() for kk, v in h.items()} for h in hops_out]
    bank.close()
    return res


@pytest.mark.parametrize("name", list(CASES))
def test_interleave_hops_against_the_oracle(name):
    w, hops = CASES[name]
    g = _run(w, hops)
    inp = P.oracle_inputs(w)
    lens, k, n = w.doc_lens(), w.top_k, w.n_docs
    off = O.doc_offsets(lens)
    B, Hkv, nblk = w.batch, w.n_kv_heads, w.q_tokens // w.route_block
    K_r, chunk_doc = zip(*[O.build_routing_keys(inp["R"][h], lens) for h in range(Hkv)])
    dkey = [[O.doc_routing_key(inp["R"][h, off[j]:off[j + 1]]) for j in range(n)] for h in range(Hkv)]
    tol = P.OUT_MAX_ABS_F32 if w.dtype == "f32" else P.OUT_MAX_ABS
    for b in range(B):
        for h in range(Hkv):
            qb = O.block_mean_query(inp["Qr"][b, h], w.route_block)
            for blk in range(nblk):
                q = qb[blk]
                for t in range(hops):
                    ctx = g[t]["ctx"][b, blk, h]
                    assert len(set(ctx.tolist())) == ctx.size and ctx.min() >= 0 and ctx.max() < n
                    if t:
                        np.testing.assert_array_equal(ctx[:t * k], g[t - 1]["ctx"][b, blk, h])
                    new = ctx[t * k:]
                    sc = O.route_doc_scores(q, K_r[h], chunk_doc[h], n)
                    sc_ex = sc.copy()
                    sc_ex[ctx[:t * k]] = -np.inf
                    want = O.select_top_k(sc_ex, k)
                    np.testing.assert_allclose(g[t]["tsc"][b, blk, h], sc[new], rtol=0, atol=P.SCORE_ABS)
                    if set(want.tolist()) != set(new.tolist()):
                        srt = np.sort(sc_ex)[::-1]
                        kth = srt[k - 1]
                        assert kth - srt[k] < P.TIE, f"hop {t}: new documents differ without a near tie"
                        diff = set(want.tolist()) ^ set(new.tolist())
                        assert all(abs(sc[j] - kth) < P.TIE for j in diff)
                    # the next query: the oracle's update by the documents the GPU took
                    q_next = O.interleave_next_query(q, [dkey[h][j] for j in new])
                    got = g[t]["q_out"][b, h, blk]
                    assert np.abs(got - q_next).max() <= 2e-5 * max(1.0, np.abs(q_next).max()), (b, h, blk, t)
                    q = q_next
    for t in range(hops):
        ref = O.forward(inp, lens, (t + 1) * k, w.route_block, w.rope_base, selection=g[t]["ctx"])
        P.check_out(g[t]["out"], ref["out"], max_abs=tol)
    if hops * k == n:
        from tests.test_oracle_pins import _dense_reference
        dense = _dense_reference(inp, list(lens), O.k_offset(n, lens), w.rope_base)
        P.check_out(g[-1]["out"], dense, max_abs=tol)


def test_interleave_argument_checks():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = CASES["decode"][0]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, 1)
    ctx = torch.zeros((w.batch, 1, w.n_kv_heads, 38), dtype=torch.int32, device="cuda")
    out = torch.empty((w.batch, 1, w.n_kv_heads, 42), dtype=torch.int32, device="cuda")
    # 38 documents in the context + 4 new > 40 documents
    assert msa.msa_interleave_route(bank.handle, qry, 4, 0, ctx.data_ptr(), 38, out.data_ptr(), 0, 0,
                                    check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_interleave_route(bank.handle, qry, 4, 0, 0, 2, out.data_ptr(), 0, 0,
                                    check=False) == msa.MSA_ERR_INVALID_ARG
    # a context index outside the bank raises the device flag
    ctx2 = torch.full((w.batch, 1, w.n_kv_heads, 2), 99, dtype=torch.int32, device="cuda")
    out2 = torch.empty((w.batch, 1, w.n_kv_heads, 6), dtype=torch.int32, device="cuda")
    assert msa.msa_interleave_route(bank.handle, qry, 4, 0, ctx2.data_ptr(), 2, out2.data_ptr(), 0, 0,
                                    check=False) == msa.MSA_OK
    assert bank.device_error() == msa.MSA_ERR_INVALID_ARG
    assert bank.device_error() == msa.MSA_OK
    bank.close()
