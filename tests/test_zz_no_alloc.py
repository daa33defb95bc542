"""msa_route_noalloc: the routing step for callers that must not allocate device
memory while they run (a process held to a fixed device-memory budget or pool,
or a host that cannot accept the implicit device synchronisation a cudaMalloc
can bring). Its scratch is the library's fixed 4 MiB device array.

Checked through the C ABI against msa_route (the allocating entry point) on two
calls in a row, so that a second call that reuses the shared array without
clearing it would show -- on a decode shape (the router that forms q_r itself)
and on a shape with more than 16 routing rows (q_r formed first, then the
tcgen05 router); the size limit is enforced before any launch.
"""
import numpy as np
import pytest
import torch

from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu


def _bank_and_query(w):
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    keep = (K, V, Q, Qr, LK, LV)
    return bank, bank.query(Q, Qr, LK, LV, w.route_block), keep


@pytest.mark.parametrize("w", [
    # 6 routing rows of 2-token blocks: q_r formed inside the mma.sync router
    Workload("noalloc_check", 21, 3, 16, 4, 128, 70, 0, 64, 4, 2, 7, ragged=(1, 900)),
    # 3 sequences x 8 one-token routing blocks = 24 routing rows (> 16): q_r kernel, then the tcgen05 router
    Workload("noalloc_tc", 25, 3, 8, 2, 128, 40, 0, 96, 8, 1, 5, ragged=(1, 900)),
], ids=lambda w: w.name)
def test_route_noalloc_matches_route_on_two_calls(w):
    import sparse_attention_routed_b200 as msa
    bank, qry, keep = _bank_and_query(w)
    stream = torch.cuda.current_stream().cuda_stream
    idx_ref, tsc_ref, sc_ref = bank.route(qry, w.top_k)
    torch.cuda.synchronize()
    shape = tuple(idx_ref.shape)
    for _ in range(2):
        idx = torch.full(shape, -1, dtype=torch.int32, device="cuda")
        tsc = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        assert msa.msa_route_noalloc(bank.handle, qry, w.top_k, 0, idx.data_ptr(), tsc.data_ptr(), stream,
                                     check=False) == msa.MSA_OK
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
        np.testing.assert_allclose(tsc.cpu().numpy(), tsc_ref.cpu().numpy(), rtol=0, atol=P.SCORE_ABS)
    # with caller-provided document scores the scratch holds only q_r
    sc = torch.full(tuple(sc_ref.shape), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full(shape, -1, dtype=torch.int32, device="cuda")
    assert msa.msa_route_noalloc(bank.handle, qry, w.top_k, sc.data_ptr(), idx.data_ptr(), 0, stream,
                                 check=False) == msa.MSA_OK
    torch.cuda.synchronize()
    np.testing.assert_allclose(sc.cpu().numpy(), sc_ref.cpu().numpy(), rtol=0, atol=P.SCORE_ABS)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
    assert bank.device_error() == 0
    bank.close()


def test_route_noalloc_rejects_steps_beyond_its_scratch():
    import sparse_attention_routed_b200 as msa
    # 16 rows x 8 KV heads x 8192 documents of scores = 4 MiB, plus q_r: over the limit
    w = Workload("noalloc_limit", 22, 16, 8, 8, 128, 8192, 1, 1, 1, 1, 4)
    bank, qry, keep = _bank_and_query(w)
    stream = torch.cuda.current_stream().cuda_stream
    idx = torch.empty((16, 1, 8, 4), dtype=torch.int32, device="cuda")
    assert msa.msa_route_noalloc(bank.handle, qry, 4, 0, idx.data_ptr(), 0, stream,
                                 check=False) == msa.MSA_ERR_UNSUPPORTED
    sc = torch.empty((16, 1, 8, 8192), dtype=torch.float32, device="cuda")
    assert msa.msa_route_noalloc(bank.handle, qry, 4, sc.data_ptr(), idx.data_ptr(), 0, stream,
                                 check=False) == msa.MSA_OK
    idx_ref, _, _ = bank.route(qry, 4)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
    bank.close()
