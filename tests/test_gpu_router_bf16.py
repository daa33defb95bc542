"""The reduced-precision router (msa_set_router_precision(MSA_KR_BF16)): only the
bf16 high part of the normalised K_r is read. Against the oracle's bf16-key
cosine (chunk_cosines_bf16_keys): scores within the router tolerance, the top-k
exact on the GPU's own scores and equal to the oracle's up to near ties, and the
attention over the selection unchanged. Both routers: the mma.sync one (at most
16 routing rows per KV head) and the tcgen05 one (more rows)."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    # 8 decode rows per KV head: mma.sync router, ragged documents
    "kr_bf16_decode": Workload("kr_bf16_decode", 81, 8, 8, 2, 128, 40, 0, 200, 1, 1, 5, ragged=(1, 900)),
    # 64 routing rows per KV head: tcgen05 router, 4-token blocks
    "kr_bf16_tc": Workload("kr_bf16_tc", 82, 2, 8, 2, 128, 30, 0, 300, 128, 4, 4, ragged=(1, 900)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_router_bf16_keys(name):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = CASES[name]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    _, _, full = bank.route(qry, w.top_k)
    bank.set_router_precision(msa.MSA_KR_BF16)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    idx2, out2 = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    full, idx, tsc, scores = (t.cpu().numpy() for t in (full, idx, tsc, scores))
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, router_keys="bf16")
    rows = scores.reshape(-1, w.n_docs)
    P.check_scores(rows, ref["doc_scores"].reshape(-1, w.n_docs))
    P.check_topk(idx.reshape(-1, w.top_k), tsc.reshape(-1, w.top_k), rows,
                 ref["doc_scores"].reshape(-1, w.n_docs), w.top_k)
    # the variant is a different score (within its rounding bound of the full-precision router)
    gap = np.abs(rows - full.reshape(-1, w.n_docs)).max()
    assert 0 < gap <= 2.0 ** -8
    ref2 = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=idx)
    P.check_out(out.cpu().numpy(), ref2["out"])
    np.testing.assert_array_equal(idx2.cpu().numpy(), idx)
    np.testing.assert_array_equal(out2.cpu().numpy(), out.cpu().numpy())
    # back to full precision
    bank.set_router_precision(msa.MSA_KR_F32)
    _, _, again = bank.route(qry, w.top_k)
    np.testing.assert_array_equal(again.cpu().numpy(), full)
    with pytest.raises(msa.MsaError):
        bank.set_router_precision(7)
    bank.close()
