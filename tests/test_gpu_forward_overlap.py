"""msa_forward on decode shapes launches the top-k and the attention as programmatic
dependents, and the attention's local-context CTAs start before the selection
exists. They must still see inputs that a kernel wrote just before the call on the
same stream: steps run back to back on a side stream, each preceded by a kernel
that writes new queries, routing queries and local K/V, with no synchronisation in
between; every step's selection and output must equal, bit for bit, msa_route +
msa_attend on the same inputs afterwards."""
import numpy as np
import pytest
import torch

from synth import Workload

pytestmark = pytest.mark.gpu

CASES = {
    # 4 query heads per KV head, 1-token blocks: many splits, local splits of their own
    "gqa4": Workload("overlap_gqa4", 51, 4, 16, 4, 128, 64, 2048, 1024, 1, 1, 8),
    # 4-token blocks, ragged documents, a short local context
    "blocks": Workload("overlap_blocks", 52, 2, 8, 2, 128, 40, 0, 96, 8, 4, 5, ragged=(1, 900)),
    "d64": Workload("overlap_d64", 53, 3, 8, 8, 64, 30, 700, 300, 1, 1, 6),
}


@pytest.mark.parametrize("name", list(CASES))
def test_back_to_back_steps_see_fresh_inputs(name):
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, fill_normal, query_tensors
    w = CASES[name]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    bank.reserve(qry, w.top_k)
    torch.cuda.synchronize()
    nblk = w.q_tokens // w.route_block
    steps = 6
    idx = [torch.empty((w.batch, nblk, w.n_kv_heads, w.top_k), dtype=torch.int32, device="cuda")
           for _ in range(steps)]
    out = [torch.empty((w.batch, w.n_q_heads, w.q_tokens, w.head_dim), dtype=torch.float32, device="cuda")
           for _ in range(steps)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for s in range(steps):
            for t, tid in ((Q, 200), (Qr, 201), (LK, 202), (LV, 203)):
                fill_normal(t, w.seed + 77 * (s + 1), tid)
            bank.forward(qry, w.top_k, idx[s], out[s], stream=side)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    for s in range(steps):
        for t, tid in ((Q, 200), (Qr, 201), (LK, 202), (LV, 203)):
            fill_normal(t, w.seed + 77 * (s + 1), tid)
        ref_idx, _, _ = bank.route(qry, w.top_k)
        ref_out = bank.attend(qry, w.top_k, ref_idx)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx[s].cpu().numpy(), ref_idx.cpu().numpy(), err_msg=f"step {s}")
        np.testing.assert_array_equal(out[s].cpu().numpy(), ref_out.cpu().numpy(), err_msg=f"step {s}")
    assert bank.device_error() == 0
    bank.close()
