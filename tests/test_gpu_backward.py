"""Backward of the routed attention (msa_attend_backward) against the oracle's
backward, on the GPU's own selection: gradients of sum(d_out * out) with respect
to the queries, the local keys and values, and the bank keys (before Parallel
RoPE) and values.

Tolerance: the kernels take bf16 operands (RoPE'd queries and keys, values, d_out,
P and dS) with fp32 accumulation, so every gradient carries the relative error of
a few bf16 roundings (2^-9 each) summed over many terms; each gradient tensor must
be within 2e-2 relative L2 of the fp64 oracle and within 4e-2 of its largest
magnitude element by element."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    # decode kernel shapes, ragged documents, G = 4
    "bwd_decode": Workload("bwd_decode", 61, 2, 8, 2, 128, 12, 0, 150, 1, 1, 3, ragged=(1, 400)),
    # 256-row problems (4 heads x 64 tokens): several dQ CTAs and two dK/dV row slices
    "bwd_prefill": Workload("bwd_prefill", 62, 1, 8, 2, 128, 8, 0, 320, 128, 64, 2, ragged=(40, 300)),
    # routing blocks of 8 tokens, G = 2, a ragged local tail
    "bwd_blocks": Workload("bwd_blocks", 63, 2, 4, 2, 128, 10, 0, 77, 16, 8, 4, ragged=(1, 250)),
    # head_dim 64, every document selected
    "bwd_d64_all": Workload("bwd_d64_all", 64, 1, 4, 1, 64, 6, 0, 40, 4, 2, 6, ragged=(5, 90)),
    # one-token documents, Lc = Tq = 1
    "bwd_tiny_docs": Workload("bwd_tiny_docs", 65, 2, 2, 2, 128, 4, 0, 1, 1, 1, 2, ragged=(1, 3)),
    # key-tile tcgen05 dK/dV: 128-token routing blocks, G = 2, queries after 44 local tokens
    # (local tiles that only some blocks reach, a ragged third local tile)
    "bwd_tc_bq128": Workload("bwd_tc_bq128", 67, 1, 4, 2, 128, 6, 0, 300, 256, 128, 3, ragged=(60, 500)),
    # key-tile tcgen05 dK/dV: 6 problems per KV head choosing 2 of 3 documents, so
    # most key tiles gather the rows of several problems
    "bwd_tc_hot": Workload("bwd_tc_hot", 68, 2, 8, 2, 128, 3, 0, 192, 192, 64, 2, ragged=(100, 400)),
}


def _close(gpu, ref, name):
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-12)
    rel_l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    worst = np.abs(gpu - ref).max() / scale
    assert rel_l2 <= 2e-2 and worst <= 4e-2, f"{name}: rel L2 {rel_l2:.2e}, max {worst:.2e} of max |ref|"


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, normal, query_tensors
    w = CASES[name]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    d_out = normal(tuple(out.shape), w.seed, 77).float()  # bf16-exact upstream gradient
    dq = torch.empty_like(out)
    dlk = torch.empty(LK.shape, dtype=torch.float32, device="cuda")
    dlv = torch.empty(LV.shape, dtype=torch.float32, device="cuda")
    dbk = torch.zeros(K.shape, dtype=torch.float32, device="cuda")
    dbv = torch.zeros(V.shape, dtype=torch.float32, device="cuda")
    msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(), dq.data_ptr(),
                            dlk.data_ptr(), dlv.data_ptr(), dbk.data_ptr(), dbv.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    inp = P.oracle_inputs(w)
    ref = O.backward(inp, w.doc_lens(), w.top_k, w.route_block, d_out.cpu().numpy().astype(np.float64),
                     w.rope_base, selection=idx.cpu().numpy())
    _close(dq.cpu().numpy(), ref["dQ"], "dQ")
    _close(dlk.cpu().numpy(), ref["dLK"], "dLK")
    _close(dlv.cpu().numpy(), ref["dLV"], "dLV")
    _close(dbk.cpu().numpy(), ref["dK"], "dK")
    _close(dbv.cpu().numpy(), ref["dV"], "dV")
    bank.close()


@pytest.mark.parametrize("name", ["bwd_decode", "bwd_tc_hot"])
def test_backward_adds_to_the_bank_gradients_and_refuses_a_host_bank(name):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, normal, query_tensors
    w = CASES[name]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    d_out = normal(tuple(out.shape), w.seed, 78).float()
    bufs = [torch.empty_like(out), torch.empty(LK.shape, dtype=torch.float32, device="cuda"),
            torch.empty(LV.shape, dtype=torch.float32, device="cuda")]
    dbk = torch.zeros(K.shape, dtype=torch.float32, device="cuda")
    dbv = torch.zeros(V.shape, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run():
        msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(), bufs[0].data_ptr(),
                                bufs[1].data_ptr(), bufs[2].data_ptr(), dbk.data_ptr(), dbv.data_ptr(), s)

    run()
    torch.cuda.synchronize()
    once_k, once_v = dbk.clone(), dbv.clone()
    run()
    torch.cuda.synchronize()
    torch.testing.assert_close(dbk, 2 * once_k, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(dbv, 2 * once_v, rtol=1e-5, atol=1e-6)
    bank.close()
    # a pinned-host bank has no device K/V to differentiate in place
    from synth.device import host_kv_pool
    wh = Workload("bwd_host", 66, 1, 4, 2, 128, 6, 0, 64, 1, 1, 2, ragged=(10, 100), host_tier=True, kv_slabs=3)
    Kh, Vh = host_kv_pool(wh)
    _, _, Rh = bank_tensors(wh)
    hb = Bank(Kh, Vh, wh.doc_lens(), wh.rope_base, kv_location=msa.MSA_KV_PINNED_HOST, doc_rows=wh.doc_kv_rows())
    hb.build(Rh, rope=False)
    Q2, Qr2, LK2, LV2 = query_tensors(wh)
    q2 = hb.query(Q2, Qr2, LK2, LV2, wh.route_block)
    i2, o2 = hb.forward(q2, wh.top_k)
    g = torch.zeros(Kh.shape, dtype=torch.float32, device="cuda")
    st = msa.msa_attend_backward(hb.handle, q2, wh.top_k, i2.data_ptr(), o2.data_ptr(), o2.data_ptr(),
                                 LK2.data_ptr(), LV2.data_ptr(), g.data_ptr(), g.data_ptr(), s, check=False)
    assert st == msa.MSA_ERR_UNSUPPORTED
    hb.close()
