"""The fp32 path (banks of MSA_DTYPE_F32) against the oracle, element by element.

The tiny configuration is stated in fp32 ("seed 0, fp32, values N(0,1)"); its inputs
here use all 24 significant bits (synth.gaussian_f32), both sides read the same fp32
numbers, and the library keeps them in fp32 end to end: pooling, Parallel RoPE
stored in fp32, q_r, and attention on the CUDA cores with fp32 operands, products
and softmax. The output bar is 1e-4 max-abs against the fp64 oracle; K_r, router
scores and top-k use the same rules as the bf16 path. Further shapes cover GQA,
ragged documents, several routing blocks, many rows per problem (two CTAs),
top_k = n_docs (the dense special case) and more than 16 routing rows (the
tcgen05 router on fp32 q_r)."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_f32": synth.WORKLOADS["tiny_f32"],
    "f32_decode_gqa": Workload("f32_decode_gqa", 31, 2, 8, 2, 128, 24, 0, 200, 1, 1, 4, ragged=(1, 700),
                               dtype="f32"),
    # 2 heads x 16 tokens = 32 rows per problem (two CTAs), 3 routing blocks, ragged local tail
    "f32_blocks": Workload("f32_blocks", 32, 1, 4, 2, 64, 12, 0, 150, 48, 16, 3, ragged=(20, 300), dtype="f32"),
    "f32_all_docs": Workload("f32_all_docs", 33, 1, 4, 1, 64, 10, 0, 64, 4, 4, 10, ragged=(1, 90), dtype="f32"),
    # 3 sequences x 8 one-token blocks = 24 routing rows: the tcgen05 router over fp32 q_r
    "f32_route_tc": Workload("f32_route_tc", 34, 3, 4, 2, 128, 16, 0, 40, 8, 1, 3, ragged=(1, 300), dtype="f32"),
}


def run_gpu(w: Workload):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    assert K.dtype == torch.float32 and Q.dtype == torch.float32
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
    out_l = torch.empty_like(out)
    msa.msa_attend_lse(bank.handle, qry, w.top_k, idx.data_ptr(), out_l.data_ptr(), lse.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
    idx2, out2 = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = {"K_r": bank.k_r().cpu().numpy(), "K_rot": K.cpu().numpy().astype(np.float64),
           "idx": idx.cpu().numpy(), "tsc": tsc.cpu().numpy(), "scores": scores.cpu().numpy(),
           "out": out.cpu().numpy(), "out_l": out_l.cpu().numpy(), "lse": lse.cpu().numpy(),
           "idx2": idx2.cpu().numpy(), "out2": out2.cpu().numpy()}
    bank.close()
    return res


@pytest.mark.parametrize("name", list(CASES))
def test_fp32_parity(name):
    w = CASES[name]
    g = run_gpu(w)
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base)
    P.check_kr(g["K_r"], ref["K_r"])
    # Parallel RoPE stored in fp32: a few fp32 roundings of values below 6 in magnitude
    assert np.abs(g["K_rot"] - ref["K_rot"]).max() <= 1e-5
    rows = g["scores"].reshape(-1, w.n_docs)
    P.check_scores(rows, ref["doc_scores"].reshape(-1, w.n_docs))
    P.check_topk(g["idx"].reshape(-1, w.top_k), g["tsc"].reshape(-1, w.top_k), rows,
                 ref["doc_scores"].reshape(-1, w.n_docs), w.top_k)
    ref2 = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=g["idx"])
    mx, mean, rel = P.check_out(g["out"], ref2["out"], max_abs=P.OUT_MAX_ABS_F32)
    print(f"{name}: max-abs {mx:.2e} mean-abs {mean:.2e} rel-L2 {rel:.2e}")
    np.testing.assert_array_equal(g["out_l"], g["out"])
    np.testing.assert_array_equal(g["idx2"], g["idx"])
    np.testing.assert_array_equal(g["out2"], g["out"])
    # each row's log-sum-exp against the oracle's
    off = O.doc_offsets(w.doc_lens())
    G = w.n_q_heads // w.n_kv_heads
    k_off = O.k_offset(w.top_k, w.doc_lens())
    for b in range(w.batch):
        for hq in range(0, w.n_q_heads, max(1, G - 1)):
            h = hq // G
            for t in range(0, w.q_tokens, max(1, w.q_tokens // 5)):
                docs = g["idx"][b, t // w.route_block, h]
                mk = np.concatenate([ref2["K_rot"][h, off[j]:off[j + 1]] for j in docs])
                i = w.local_len - w.q_tokens + t
                want = O.routed_attention_row_lse(inp["Q"][b, hq, t], i, k_off, w.rope_base, mk, inp["LK"][b, h])
                assert abs(g["lse"][b, hq, t] - want) <= 1e-5, (b, hq, t)


def test_fp32_all_docs_equals_dense_reference():
    w = CASES["f32_all_docs"]
    g = run_gpu(w)
    from tests.test_oracle_pins import _dense_reference
    dense = _dense_reference(P.oracle_inputs(w), list(w.doc_lens()), O.k_offset(w.top_k, w.doc_lens()),
                             w.rope_base)
    P.check_out(g["out"], dense, max_abs=P.OUT_MAX_ABS_F32)


def test_fp32_backward_is_refused():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = synth.WORKLOADS["tiny_f32"]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    g = [torch.zeros_like(out), torch.zeros_like(LK), torch.zeros_like(LV), torch.zeros_like(K),
         torch.zeros_like(V)]
    st = msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(),
                                 *[t.data_ptr() for t in g], torch.cuda.current_stream().cuda_stream, check=False)
    assert st == msa.MSA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    bank.close()
