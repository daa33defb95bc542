"""CUDA path vs the CPU oracle on the same seeded inputs (small, oracle-complete cases).

Sizes span several 64-key tiles, ragged document tails, ragged local tails,
several routing blocks, GQA groups of 1, 2, 4 and 8, head_dim 64 and 128,
top_k = n_docs (the dense special case) and the one-token degenerate case.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": synth.WORKLOADS["tiny"],
    "decode_small": Workload("decode_small", 11, 2, 8, 2, 128, 48, 1024, 512, 1, 1, 4),
    "ragged_small": Workload("ragged_small", 12, 2, 16, 2, 128, 40, 0, 300, 1, 1, 5, ragged=(1, 700)),
    "blocks_small": Workload("blocks_small", 13, 1, 4, 2, 128, 24, 600, 130, 8, 4, 3),
    "d64_all_docs": Workload("d64_all_docs", 14, 3, 8, 1, 64, 20, 333, 77, 2, 2, 20),
    "one_token": Workload("one_token", 15, 1, 2, 2, 128, 3, 0, 1, 1, 1, 1, ragged=(1, 3)),
    "planted_small": Workload("planted_small", 16, 2, 8, 8, 128, 30, 0, 64, 1, 1, 4, ragged=(300, 1500),
                              planted=4),
    # many-row problems (prefill kernel): 4 heads x 64 tokens = 256 rows over 2 CTAs
    "prefill_small": Workload("prefill_small", 17, 1, 8, 2, 128, 24, 600, 256, 256, 64, 3),
    # 3 heads x 48 tokens = 144 rows (a 16-row tail CTA), ragged docs, queries not at the local start
    "prefill_ragged": Workload("prefill_ragged", 18, 2, 6, 2, 128, 20, 0, 300, 96, 48, 4, ragged=(1, 900)),
    "prefill_d64": Workload("prefill_d64", 19, 1, 4, 1, 64, 12, 0, 200, 64, 32, 12, ragged=(50, 400)),
    # more than 16 routing rows per KV head: the tcgen05 router (64 rows, ragged documents)
    "route_tc_rows": Workload("route_tc_rows", 20, 2, 8, 2, 128, 30, 0, 300, 32, 1, 5, ragged=(1, 900)),
    # 160 routing rows: two passes of the tcgen05 router (128 + 32 rows)
    "route_tc_passes": Workload("route_tc_passes", 22, 5, 4, 4, 128, 20, 520, 64, 32, 1, 3),
    # tcgen05 prefill with 128-token routing blocks and G = 1 (one 128-row CTA per problem);
    # the queries are the whole local context (Lc = Tq)
    "prefill_bq128": Workload("prefill_bq128", 23, 1, 2, 2, 128, 10, 0, 256, 256, 128, 3, ragged=(60, 700)),
    # the largest top_k (64) over 80 short documents, decode kernel with G = 2
    "topk64": Workload("topk64", 24, 2, 4, 2, 128, 80, 0, 130, 1, 1, 64, ragged=(1, 200)),
    # a long local context next to two short documents: most decode splits are the local
    # context's own (and a single document split per problem)
    "local_heavy": Workload("local_heavy", 26, 2, 8, 2, 128, 6, 100, 6000, 1, 1, 2),
}


@pytest.fixture(scope="module")
def dev():
    from synth import device  # noqa: F401  (loads the generator library)
    assert torch.cuda.is_available()
    return torch.device("cuda")


def run_gpu(w: Workload):
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    idx2, out2 = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = {"K_r": bank.k_r().cpu().numpy(), "K_rot": K.float().cpu().numpy(), "idx": idx.cpu().numpy(),
           "tsc": tsc.cpu().numpy(), "scores": scores.cpu().numpy(), "out": out.cpu().numpy(),
           "idx2": idx2.cpu().numpy(), "out2": out2.cpu().numpy()}
    bank.close()
    return res


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(dev, name):
    w = SMALL[name]
    g = run_gpu(w)
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base)
    P.check_kr(g["K_r"], ref["K_r"])
    P.check_rope_keys(g["K_rot"], ref["K_rot"])
    rows = g["scores"].reshape(-1, w.n_docs)
    P.check_scores(rows, ref["doc_scores"].reshape(-1, w.n_docs))
    P.check_topk(g["idx"].reshape(-1, w.top_k), g["tsc"].reshape(-1, w.top_k), rows,
                 ref["doc_scores"].reshape(-1, w.n_docs), w.top_k)
    # attention over the GPU's own (validated) selection
    ref2 = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=g["idx"])
    P.check_out(g["out"], ref2["out"])
    # msa_forward = msa_route + msa_attend, bit for bit
    np.testing.assert_array_equal(g["idx2"], g["idx"])
    np.testing.assert_array_equal(g["out2"], g["out"])
    if w.planted:
        targets = synth.planted_targets(w.seed, w.batch, w.n_docs, w.planted)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                t = targets[b, h % w.planted]
                assert (t in g["idx"][b, 0, h]) == (t in ref["topk"][b, 0, h])


def test_all_docs_equals_dense_reference(dev):
    """top_k = n_docs: the GPU result equals dense attention over the whole bank."""
    w = SMALL["d64_all_docs"]
    g = run_gpu(w)
    inp = P.oracle_inputs(w)
    from tests.test_oracle_pins import _dense_reference
    dense = _dense_reference(inp, list(w.doc_lens()), O.k_offset(w.top_k, w.doc_lens()), w.rope_base)
    P.check_out(g["out"], dense)


def test_invalid_queries_rejected(dev):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = SMALL["decode_small"]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens())
    bank.build(R)
    idx = torch.zeros((w.batch, 1, w.n_kv_heads, w.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((w.batch, w.n_q_heads, 1, w.head_dim), dtype=torch.float32, device="cuda")
    p = msa.ptr
    good = dict(batch=w.batch, n_q_heads=w.n_q_heads, q_tokens=1, local_len=w.local_len, route_block=1)
    for bad in (dict(batch=0), dict(n_q_heads=7), dict(q_tokens=w.local_len + 1), dict(route_block=0),
                dict(q_tokens=3, route_block=2)):
        kw = dict(good)
        kw.update(bad)
        q = msa.make_query(kw["batch"], kw["n_q_heads"], kw["q_tokens"], kw["local_len"], kw["route_block"],
                           p(Q), p(Qr), p(LK), p(LV))
        assert msa.msa_forward(bank.handle, q, w.top_k, p(idx), p(out), check=False) == msa.MSA_ERR_INVALID_ARG
    q = bank.query(Q, Qr, LK, LV, 1)
    for k in (0, w.n_docs + 1):
        assert msa.msa_forward(bank.handle, q, k, p(idx), p(out), check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_forward(bank.handle, q, 65, p(idx), p(out), check=False) in (
        msa.MSA_ERR_INVALID_ARG, msa.MSA_ERR_UNSUPPORTED)
    # an out-of-range selection index is reported through the device error flag
    idx[0, 0, 0, 0] = w.n_docs + 5
    assert msa.msa_attend(bank.handle, q, w.top_k, p(idx), p(out), check=False) == msa.MSA_OK
    assert bank.device_error() == msa.MSA_ERR_INVALID_ARG
    assert bank.device_error() == msa.MSA_OK
    bank.close()
