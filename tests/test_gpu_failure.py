"""Failure detection on the GPU without a fault: a bounded device wait that
nothing satisfies expires, the kernel returns, the host reads MSA_ERR_TIMEOUT
from the device error flag, and the same context then runs a correct step."""
import time

import pytest
import torch

import synth
from oracle import msa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_stays_usable():
    from sparse_attention_routed_b200 import MSA_ERR_TIMEOUT, MSA_OK, msa_check_wait_timeout
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = synth.WORKLOADS["tiny"]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    torch.cuda.synchronize()
    assert bank.device_error() == MSA_OK

    t0 = time.perf_counter()
    msa_check_wait_timeout(bank.handle, torch.cuda.current_stream().cuda_stream)
    status = bank.device_error()  # synchronises the stream
    waited = time.perf_counter() - t0
    assert status == MSA_ERR_TIMEOUT
    assert bank.device_error() == MSA_OK  # reading the flag cleared it
    print(f"bounded wait gave up after {waited:.3f} s")
    assert waited < 60.0

    # the context survived: a full step still matches the oracle
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == MSA_OK
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=idx.cpu().numpy())
    P.check_out(out.cpu().numpy(), ref["out"])

    # the allocation-free router raises and clears the same flag: after another
    # expired wait it reads MSA_ERR_TIMEOUT once, then routes exactly as msa_route
    from sparse_attention_routed_b200 import msa_route_noalloc
    msa_check_wait_timeout(bank.handle, torch.cuda.current_stream().cuda_stream)
    assert bank.device_error() == MSA_ERR_TIMEOUT
    idx2 = torch.full_like(idx, -1)
    msa_route_noalloc(bank.handle, qry, w.top_k, 0, idx2.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)
    assert bank.device_error() == MSA_OK
    assert torch.equal(idx2, idx)
    bank.close()
