"""Pinned-host K/V tier: K/V in pinned host memory, the selected documents'
slabs copied into a device staging pool each step. Checked against the CPU
oracle, and bit for bit against a device-resident bank over the same K/V."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

HOST = {
    # decode, G = 4, ragged documents, 5 slabs for 40 documents (aliased pool)
    "host_decode": Workload("host_decode", 31, 2, 8, 2, 128, 40, 0, 300, 1, 1, 6, ragged=(1, 700),
                            host_tier=True, kv_slabs=5),
    # planted targets, G = 8
    "host_planted": Workload("host_planted", 32, 2, 16, 2, 128, 30, 0, 100, 1, 1, 4, ragged=(300, 1500),
                             planted=4, host_tier=True, kv_slabs=7),
    # 256-row problems (tcgen05 prefill) reading the staging pool
    "host_prefill": Workload("host_prefill", 33, 1, 8, 2, 128, 16, 0, 256, 128, 64, 3, ragged=(100, 900),
                             host_tier=True, kv_slabs=4),
    # 5 sequences: msa_forward runs micro-batches of 2, 2 and 1 sequences; 12 equal-length
    # documents over 6 slabs, so sequences share slabs across micro-batches and slabs that
    # are neighbours in host memory are copied as one
    "host_micro": Workload("host_micro", 34, 5, 8, 2, 128, 12, 300, 200, 1, 1, 4, host_tier=True, kv_slabs=6),
}


def _run(w, host: bool, fetch=None):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, host_kv_pool, query_tensors
    if host:
        K, V = host_kv_pool(w)
        _, _, R = bank_tensors(w)
        kv_loc = msa.MSA_KV_PINNED_HOST
    else:
        K, V, R = bank_tensors(w)
        slabs = Bank(K, V, [w.max_len] * w.kv_slabs, w.rope_base)   # same RoPE'd slabs, on the device
        slabs.build(None)
        torch.cuda.synchronize()
        slabs.close()
        kv_loc = msa.MSA_KV_DEVICE
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base, kv_location=kv_loc, doc_rows=w.doc_kv_rows())
    bank.build(R, rope=False)
    if fetch is not None:
        bank.set_host_fetch(fetch)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    idx2, out2 = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = dict(idx=idx.cpu().numpy(), tsc=tsc.cpu().numpy(), scores=scores.cpu().numpy(), out=out.cpu().numpy(),
               idx2=idx2.cpu().numpy(), out2=out2.cpu().numpy())
    # an out-of-range selection index is caught on the host before any copy
    bad = idx.clone()
    bad[0, 0, 0, 0] = w.n_docs
    if host:
        st = msa.msa_attend(bank.handle, qry, w.top_k, bad.data_ptr(), out.data_ptr(),
                            torch.cuda.current_stream().cuda_stream, check=False)
        res["bad_status"] = st
        res["fetch"] = bank.host_fetch()
        res["stats"] = bank.cache_stats()
    bank.close()
    return res


@pytest.mark.parametrize("name", list(HOST))
def test_host_tier_parity(name):
    w = HOST[name]
    g = _run(w, host=True)
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base)
    rows = g["scores"].reshape(-1, w.n_docs)
    P.check_scores(rows, ref["doc_scores"].reshape(-1, w.n_docs))
    P.check_topk(g["idx"].reshape(-1, w.top_k), g["tsc"].reshape(-1, w.top_k), rows,
                 ref["doc_scores"].reshape(-1, w.n_docs), w.top_k)
    ref2 = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=g["idx"])
    P.check_out(g["out"], ref2["out"])
    # msa_forward pipelines micro-batches of sequences (its split-KV partition may differ
    # from msa_attend's on the whole batch, so its output is checked against the oracle)
    np.testing.assert_array_equal(g["idx2"], g["idx"])
    P.check_out(g["out2"], ref2["out"])
    import sparse_attention_routed_b200 as msa
    assert g["bad_status"] == msa.MSA_ERR_INVALID_ARG


def test_host_tier_equals_device_bank():
    w = HOST["host_decode"]
    gh = _run(w, host=True)
    gd = _run(w, host=False)
    np.testing.assert_array_equal(gh["idx"], gd["idx"])
    np.testing.assert_array_equal(gh["out"], gd["out"])


@pytest.mark.parametrize("name", list(HOST))
def test_host_fetch_transports_agree(name):
    """The SM gather (the default: torch's pinned memory is mapped) and the copy-engine
    transfers stage the same bytes: routing and outputs bit for bit equal."""
    import sparse_attention_routed_b200 as msa
    w = HOST[name]
    gd = _run(w, host=True)
    assert gd["fetch"] == msa.MSA_FETCH_SM_GATHER
    gc = _run(w, host=True, fetch=msa.MSA_FETCH_COPY_ENGINE)
    assert gc["fetch"] == msa.MSA_FETCH_COPY_ENGINE
    for key in ("idx", "out", "idx2", "out2"):
        np.testing.assert_array_equal(gd[key], gc[key], err_msg=key)
    assert gd["bad_status"] == gc["bad_status"] == msa.MSA_ERR_INVALID_ARG


def test_host_fetch_arguments():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors
    w = HOST["host_decode"]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base, doc_rows=w.doc_kv_rows())
    assert msa.msa_set_host_fetch(bank.handle, msa.MSA_FETCH_SM_GATHER, check=False) == msa.MSA_ERR_INVALID_ARG
    bank.close()
    from synth.device import host_kv_pool
    Kh, Vh = host_kv_pool(w)
    hb = Bank(Kh, Vh, w.doc_lens(), w.rope_base, kv_location=msa.MSA_KV_PINNED_HOST, doc_rows=w.doc_kv_rows())
    assert msa.msa_set_host_fetch(hb.handle, 2, check=False) == msa.MSA_ERR_INVALID_ARG
    hb.set_host_fetch(msa.MSA_FETCH_COPY_ENGINE)
    assert hb.host_fetch() == msa.MSA_FETCH_COPY_ENGINE
    hb.set_host_fetch(msa.MSA_FETCH_SM_GATHER)
    assert hb.host_fetch() == msa.MSA_FETCH_SM_GATHER
    hb.close()


def test_unmapped_host_kv_falls_back_to_copy_engines():
    """Host K/V that is not page-locked (so not mapped for the device): the bank moves
    its slabs with copy-engine transfers, refuses the SM gather, and attends exactly as
    over page-locked K/V."""
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, host_kv_pool, query_tensors
    w = HOST["host_decode"]
    Kp, Vp = host_kv_pool(w)
    Ku, Vu = Kp.clone(), Vp.clone()          # ordinary (pageable) host memory
    assert not Ku.is_pinned()
    _, _, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    outs = []
    for K, V in ((Kp, Vp), (Ku, Vu)):
        bank = Bank(K, V, w.doc_lens(), w.rope_base, kv_location=msa.MSA_KV_PINNED_HOST, doc_rows=w.doc_kv_rows())
        bank.build(R, rope=False)
        qry = bank.query(Q, Qr, LK, LV, w.route_block)
        idx, out = bank.forward(qry, w.top_k)
        torch.cuda.synchronize()
        assert bank.device_error() == 0
        outs.append((bank.host_fetch(), idx.cpu().numpy(), out.cpu().numpy()))
        if K is Ku:
            assert msa.msa_set_host_fetch(bank.handle, msa.MSA_FETCH_SM_GATHER, check=False) == msa.MSA_ERR_UNSUPPORTED
        bank.close()
    assert outs[0][0] == msa.MSA_FETCH_SM_GATHER and outs[1][0] == msa.MSA_FETCH_COPY_ENGINE
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    np.testing.assert_array_equal(outs[0][2], outs[1][2])
