"""msa_attend_lse and msa_attend_backward_saved: the forward's log-sum-exp against
the oracle's (routed_attention_row_lse) on every kernel family -- decode, the
tcgen05 prefill and the mma.sync prefill --, msa_attend_lse's output bit for bit
msa_attend's, and the backward given the saved state equal to the backward that
recomputes it."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "saved_decode": Workload("saved_decode", 91, 2, 8, 2, 128, 12, 0, 150, 1, 1, 3, ragged=(1, 400)),
    "saved_prefill_tc": Workload("saved_prefill_tc", 92, 1, 8, 2, 128, 8, 0, 320, 128, 64, 2, ragged=(40, 300)),
    "saved_prefill_mma": Workload("saved_prefill_mma", 93, 2, 6, 2, 128, 10, 0, 200, 96, 48, 3, ragged=(1, 500)),
}
LSE_ABS = 1e-2   # logits from bf16 RoPE'd queries and keys: a few 2^-9 roundings


@pytest.mark.parametrize("name", list(CASES))
def test_lse_and_saved_backward(name):
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
    s = torch.cuda.current_stream().cuda_stream
    out2 = torch.empty_like(out)
    lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
    msa.msa_attend_lse(bank.handle, qry, w.top_k, idx.data_ptr(), out2.data_ptr(), lse.data_ptr(), s)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    assert torch.equal(out, out2)
    # the log-sum-exp of every row against the oracle's, over the GPU's selection
    inp = P.oracle_inputs(w)
    off = O.doc_offsets(w.doc_lens())
    k_off = O.k_offset(w.top_k, w.doc_lens())
    G = w.n_q_heads // w.n_kv_heads
    sel = idx.cpu().numpy()
    got = lse.cpu().numpy()
    ref = np.empty_like(got, dtype=np.float64)
    for b in range(w.batch):
        for hq in range(w.n_q_heads):
            h = hq // G
            for t in range(w.q_tokens):
                docs = sel[b, t // w.route_block, h]
                mk = np.concatenate([O.parallel_rope_bank(inp["K"][h, off[j]:off[j + 1]], [off[j + 1] - off[j]],
                                                          w.rope_base) for j in docs])
                ref[b, hq, t] = O.routed_attention_row_lse(inp["Q"][b, hq, t], w.local_len - w.q_tokens + t, k_off,
                                                           w.rope_base, mk, inp["LK"][b, h])
    err = np.abs(got - ref).max()
    assert err <= LSE_ABS, f"log-sum-exp error {err:.3e}"
    # backward with the saved state equals the backward that recomputes it
    d_out = normal(tuple(out.shape), w.seed, 77).float()

    def grads(saved):
        g = [torch.empty_like(out), torch.empty(LK.shape, dtype=torch.float32, device="cuda"),
             torch.empty(LV.shape, dtype=torch.float32, device="cuda"),
             torch.zeros(K.shape, dtype=torch.float32, device="cuda"),
             torch.zeros(V.shape, dtype=torch.float32, device="cuda")]
        if saved:
            msa.msa_attend_backward_saved(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                          d_out.data_ptr(), *[x.data_ptr() for x in g], s)
        else:
            msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(),
                                    *[x.data_ptr() for x in g], s)
        torch.cuda.synchronize()
        assert bank.device_error() == 0
        return g

    a, b = grads(False), grads(True)
    for x, y, nm in zip(a, b, ["dQ", "dLK", "dLV", "dK", "dV"]):
        torch.testing.assert_close(y, x, rtol=1e-6, atol=1e-7, msg=lambda m: f"{nm}: {m}")
    st = msa.msa_attend_backward_saved(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(), 0,
                                       d_out.data_ptr(), *[x.data_ptr() for x in a], s, check=False)
    assert st == msa.MSA_ERR_INVALID_ARG
    bank.close()
