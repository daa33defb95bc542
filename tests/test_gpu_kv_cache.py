"""Device-resident slab cache of the pinned-host K/V tier (msa_set_kv_cache):
outputs equal the uncached host tier bit for bit, resident slabs are not copied
again, evictions keep every step correct, and a cache too small for one step's
selection is refused."""
import numpy as np
import pytest
import torch

from synth import Workload

pytestmark = pytest.mark.gpu

# 5 sequences, 2 KV heads, 40 documents of 300 tokens over 6 pinned slabs, top 4:
# at most 40 distinct (document, head) slabs per step, 80 in all
W = Workload("cache_case", 51, 5, 8, 2, 128, 40, 300, 200, 1, 1, 4, host_tier=True, kv_slabs=6)


def _banks(n_slots):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, host_kv_pool
    Kh, Vh = host_kv_pool(W)
    _, _, R = bank_tensors(W)
    banks = []
    for _ in range(2):
        b = Bank(Kh, Vh, W.doc_lens(), W.rope_base, kv_location=msa.MSA_KV_PINNED_HOST, doc_rows=W.doc_kv_rows())
        b.build(R, rope=False)
        banks.append(b)
    slot_bytes = 2 * W.max_len * W.head_dim * 2
    banks[1].set_kv_cache(n_slots * slot_bytes)
    return banks, (Kh, Vh)


def _query(bank, step):
    from synth.device import fill_normal, query_tensors
    Q, Qr, LK, LV = query_tensors(W)
    if step:
        for t, tid in ((Q, 200), (Qr, 201), (LK, 202), (LV, 203)):
            fill_normal(t, W.seed + 977 * step, tid)
    return bank.query(Q, Qr, LK, LV, W.route_block), (Q, Qr, LK, LV)


def test_resident_slabs_are_not_copied_again():
    (plain, cached), keep = _banks(60)
    q0, k0 = _query(plain, 0)
    q1, k1 = _query(cached, 0)
    idx_r, out_r = plain.forward(q0, W.top_k)
    torch.cuda.synchronize()
    for rep in range(2):
        idx, out = cached.forward(q1, W.top_k)
        torch.cuda.synchronize()
        st = cached.cache_stats()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_r.cpu().numpy())
        np.testing.assert_array_equal(out.cpu().numpy(), out_r.cpu().numpy())
        assert st["slabs"] > 0
        if rep == 0:
            assert st["hits"] == 0 and st["bytes_copied"] > 0
        else:
            assert st["hits"] == st["slabs"] and st["bytes_copied"] == 0
    # msa_attend on the same selection reads the resident slabs as well
    out2 = cached.attend(q1, W.top_k, idx)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out2.cpu().numpy(), plain.attend(q0, W.top_k, idx_r).cpu().numpy())
    assert cached.cache_stats()["bytes_copied"] == 0
    assert plain.device_error() == 0 and cached.device_error() == 0
    for b in (plain, cached):
        b.close()


@pytest.mark.parametrize("fetch", [1, 0], ids=["sm_gather", "copy_engine"])
def test_evictions_keep_every_step_correct(fetch):
    (plain, cached), keep = _banks(44)  # room for any one step, not for the steps' union
    cached.set_host_fetch(fetch)         # the uncached bank keeps the default SM gather
    hits = copied = 0
    for step in range(6):
        q0, k0 = _query(plain, step)
        q1, k1 = _query(cached, step)
        idx_r, out_r = plain.forward(q0, W.top_k)
        idx, out = cached.forward(q1, W.top_k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_r.cpu().numpy())
        np.testing.assert_array_equal(out.cpu().numpy(), out_r.cpu().numpy())
        st = cached.cache_stats()
        hits += st["hits"]
        copied += st["bytes_copied"] > 0
    assert hits > 0 and copied > 1
    assert plain.device_error() == 0 and cached.device_error() == 0
    for b in (plain, cached):
        b.close()


def test_cache_smaller_than_one_step_is_refused():
    import sparse_attention_routed_b200 as msa
    (plain, cached), keep = _banks(60)
    cached.set_kv_cache(3 * 2 * W.max_len * W.head_dim * 2)  # 3 slots
    q1, k1 = _query(cached, 0)
    idx = torch.empty((W.batch, 1, W.n_kv_heads, W.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((W.batch, W.n_q_heads, 1, W.head_dim), dtype=torch.float32, device="cuda")
    st = msa.msa_forward(cached.handle, q1, W.top_k, idx.data_ptr(), out.data_ptr(),
                         torch.cuda.current_stream().cuda_stream, check=False)
    assert st == msa.MSA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    # a device-tier bank has no host tier to cache
    assert msa.msa_set_kv_cache(None, 0, check=False) == msa.MSA_ERR_INVALID_ARG
    for b in (plain, cached):
        b.close()


def test_device_bank_refuses_a_cache():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors
    K, V, R = bank_tensors(W)
    b = Bank(K, V, W.doc_lens(), W.rope_base, doc_rows=W.doc_kv_rows())
    assert msa.msa_set_kv_cache(b.handle, 1 << 20, check=False) == msa.MSA_ERR_INVALID_ARG
    b.close()
