"""A routed step captured into a CUDA graph after msa_reserve: replays with new
inputs written into the captured buffers give, bit for bit, what an eager
msa_forward gives on the same inputs (decode kernel and tcgen05 prefill kernel)."""
import numpy as np
import pytest
import torch

from synth import Workload

pytestmark = pytest.mark.gpu

CASES = {
    "graph_decode": Workload("graph_decode", 41, 3, 8, 2, 128, 40, 0, 300, 1, 1, 6, ragged=(1, 700)),
    "graph_prefill": Workload("graph_prefill", 42, 1, 8, 2, 128, 16, 0, 256, 128, 64, 3, ragged=(100, 900)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_captured_step_matches_eager(name):
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, fill_normal, query_tensors
    w = CASES[name]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    bank.reserve(qry, w.top_k)
    nblk = w.q_tokens // w.route_block
    idx = torch.empty((w.batch, nblk, w.n_kv_heads, w.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((w.batch, w.n_q_heads, w.q_tokens, w.head_dim), dtype=torch.float32, device="cuda")
    bank.forward(qry, w.top_k, idx, out)  # warm-up outside the capture
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bank.forward(qry, w.top_k, idx, out)
    torch.cuda.synchronize()

    for step in range(3):
        # new inputs in the captured buffers (another seeded stream each step)
        for t, tid in ((Q, 100), (Qr, 101), (LK, 102), (LV, 103)):
            fill_normal(t, w.seed + 1000 * (step + 1), tid)
        g.replay()
        torch.cuda.synchronize()
        got_idx, got_out = idx.clone(), out.clone()
        ref_idx, ref_out = bank.forward(qry, w.top_k)
        torch.cuda.synchronize()
        assert bank.device_error() == 0
        np.testing.assert_array_equal(got_idx.cpu().numpy(), ref_idx.cpu().numpy())
        np.testing.assert_array_equal(got_out.cpu().numpy(), ref_out.cpu().numpy())
        assert np.isfinite(got_out.cpu().numpy()).all()
    del g
    bank.close()
