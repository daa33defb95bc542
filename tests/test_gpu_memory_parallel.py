"""Memory Parallel on one GPU: a bank split into 2-5 document shards (each its own
bank, as each would be on its own device), routed, merged and attended through the
C ABI, against the single bank and the oracle.

* The merged selection equals the single bank's msa_route bit for bit (each shard
  scores its chunks exactly as the whole bank does; the merge keeps the order).
* The merged output matches the oracle's sharded step (which equals its single-bank
  step) within the usual tolerances, and the single bank's output closely.
* Each shard's partial matches the oracle's partial (softmax and log-sum-exp over
  the keys it holds); the owner's includes the local context.
* The merge entry points alone against the oracle's merges: candidates with exact
  ties across shards, partials with empty (-inf) parts.
* fp32 shards (1e-4), pinned-host shards (bit for bit equal to device shards), and
  many-row steps on both prefill kernels, including CTAs that hold no key at all.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "decode_gqa": (Workload("mp_decode", 41, 3, 16, 4, 128, 37, 0, 300, 1, 1, 6, ragged=(1, 900)), 3),
    "blocks": (Workload("mp_blocks", 42, 2, 4, 2, 128, 24, 0, 160, 8, 4, 4, ragged=(100, 700)), 2),
    "d64_many_shards": (Workload("mp_d64", 43, 2, 8, 2, 64, 40, 0, 96, 2, 2, 5, ragged=(1, 400)), 5),
    "f32": (Workload("mp_f32", 44, 2, 8, 2, 128, 20, 0, 128, 1, 1, 4, ragged=(1, 500), dtype="f32"), 4),
    # 4 heads x 64-token blocks = 256 rows per problem: the tcgen05 prefill kernel; with 3 shards
    # and top_k 2 some problems hold none of a shard's documents (CTAs with no key at all)
    "prefill_tc": (Workload("mp_prefill_tc", 47, 1, 8, 2, 128, 12, 0, 256, 128, 64, 2, ragged=(60, 300)), 3),
    # 3 heads x 48-token blocks = 144 rows: the mma.sync prefill kernel, d = 64
    "prefill_mma": (Workload("mp_prefill_mma", 48, 1, 6, 2, 64, 10, 0, 160, 96, 48, 3, ragged=(30, 400)), 2),
}


def build_shards(w, S, owner=0, host=False):
    from sparse_attention_routed_b200 import MSA_KV_PINNED_HOST
    from sparse_attention_routed_b200.parallel import shard_bank_tensors, shard_ranges
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    lens = w.doc_lens()
    ranges = shard_ranges(w.n_docs, S)
    banks, keep = [], [Q, Qr, LK, LV]
    for (lo, hi), (Ks, Vs, Rs) in zip(ranges, shard_bank_tensors(K, V, R, lens, ranges)):
        if host:
            Kd = Ks
            b = Bank(Ks, Vs, lens[lo:hi], w.rope_base)   # RoPE in place on the device, then to pinned memory
            b.build(None)
            torch.cuda.synchronize()
            b.close()
            Kh = torch.empty(Ks.shape, dtype=Ks.dtype, pin_memory=True)
            Vh = torch.empty(Vs.shape, dtype=Vs.dtype, pin_memory=True)
            Kh.copy_(Kd)
            Vh.copy_(Vs)
            bank = Bank(Kh, Vh, lens[lo:hi], w.rope_base, kv_location=MSA_KV_PINNED_HOST)
            bank.set_shard(lo, w.n_docs, int(lens.max()))
            bank.build(Rs, rope=False)
            keep += [Kh, Vh]
        else:
            bank = Bank(Ks, Vs, lens[lo:hi], w.rope_base)
            bank.set_shard(lo, w.n_docs, int(lens.max()))
            bank.build(Rs)
        keep += [Ks, Vs, Rs]
        banks.append(bank)
    queries = [b.query(Q, Qr, LK, LV, w.route_block) for b in banks]
    whole = Bank(K, V, lens, w.rope_base)
    whole.build(R)
    return banks, queries, whole, whole.query(Q, Qr, LK, LV, w.route_block), ranges, keep


@pytest.mark.parametrize("name", list(CASES))
def test_sharded_step_against_single_bank_and_oracle(name):
    from sparse_attention_routed_b200.parallel import ShardedStep
    w, S = CASES[name]
    owner = S - 1
    banks, queries, whole, wq, ranges, keep = build_shards(w, S, owner)
    idx, out, cands, partials = ShardedStep(banks, owner)(queries, w.top_k, parts=True)
    idx_ref, tsc_ref, _ = whole.route(wq, w.top_k, want_scores=False)
    _, out_ref = whole.forward(wq, w.top_k)
    torch.cuda.synchronize()
    for b in banks + [whole]:
        assert b.device_error() == 0
    idx, out, idx_ref, out_ref = (t.cpu().numpy() for t in (idx, out, idx_ref, out_ref))
    # the merged selection is the single bank's
    np.testing.assert_array_equal(idx, idx_ref)
    # each shard's candidates carry global indices inside its range
    for (lo, hi), (sc, ix) in zip(ranges, cands):
        ix = ix.cpu().numpy()
        assert ix.min() >= lo and ix.max() < hi
    inp = P.oracle_inputs(w)
    mp = O.memory_parallel_forward(inp, w.doc_lens(), w.top_k, w.route_block, S, w.rope_base, owner=owner)
    np.testing.assert_array_equal(mp["topk"], O.forward(inp, w.doc_lens(), w.top_k, w.route_block,
                                                        w.rope_base)["topk"])
    tol = P.OUT_MAX_ABS_F32 if w.dtype == "f32" else P.OUT_MAX_ABS
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=idx)
    P.check_out(out, ref["out"], max_abs=tol)
    assert np.abs(out - out_ref).max() <= tol
    # partials: shard s attends the selected documents it holds (+ the local context at the owner)
    if (idx == mp["topk"]).all():
        for s, (po, pl) in enumerate(partials):
            po, pl = po.cpu().numpy(), pl.cpu().numpy()
            fin = np.isfinite(mp["part_lse"][s])
            np.testing.assert_array_equal(np.isfinite(pl), fin)
            assert np.abs(pl[fin] - mp["part_lse"][s][fin]).max() <= (1e-5 if w.dtype == "f32" else 2e-3)
            assert np.abs(po - mp["part_out"][s]).max() <= tol
            assert not po[~fin].any()
    for b in banks + [whole]:
        b.close()


def test_pinned_host_shards_equal_device_shards():
    from sparse_attention_routed_b200.parallel import ShardedStep
    w = Workload("mp_host", 45, 2, 8, 2, 128, 30, 0, 200, 1, 1, 5, ragged=(1, 800))
    banks, queries, whole, wq, ranges, keep = build_shards(w, 3)
    hbanks, hqueries, hwhole, _, _, hkeep = build_shards(w, 3, host=True)
    idx, out = ShardedStep(banks)(queries, w.top_k)
    hidx, hout = ShardedStep(hbanks)(hqueries, w.top_k)
    torch.cuda.synchronize()
    for b in banks + hbanks:
        assert b.device_error() == 0
    assert torch.equal(idx, hidx)
    assert torch.equal(out, hout)
    for b in banks + hbanks + [whole, hwhole]:
        b.close()


def test_merge_topk_matches_the_oracle_merge():
    import sparse_attention_routed_b200 as msa
    rng = np.random.default_rng(7)
    for S, k, rows in ((2, 16, 64), (3, 5, 1000), (8, 64, 33), (64, 1, 7)):
        n = S * k * 2
        scores = rng.integers(-6, 7, (rows, n)).astype(np.float32) / 8.0   # many exact ties
        cs = np.empty((S, rows, k), np.float32)
        ci = np.empty((S, rows, k), np.int32)
        bounds = np.linspace(0, n, S + 1).astype(int)
        for s in range(S):
            lo, hi = bounds[s], bounds[s + 1]
            for r in range(rows):
                loc = O.select_top_k(scores[r, lo:hi], k)
                ci[s, r] = loc + lo
                cs[s, r] = scores[r, lo:hi][loc]
        dcs, dci = torch.from_numpy(cs).cuda(), torch.from_numpy(ci).cuda()
        idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
        sc = torch.empty((rows, k), dtype=torch.float32, device="cuda")
        msa.msa_merge_topk(S, rows, k, dcs.data_ptr(), dci.data_ptr(), idx.data_ptr(), sc.data_ptr())
        torch.cuda.synchronize()
        idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
        for r in range(rows):
            want, wsc = O.merge_candidates(list(cs[:, r]), list(ci[:, r]), k)
            np.testing.assert_array_equal(idx[r], want)
            np.testing.assert_array_equal(sc[r], wsc.astype(np.float32))


def test_merge_partials_matches_the_oracle_merge():
    import sparse_attention_routed_b200 as msa
    rng = np.random.default_rng(8)
    S, rows, d = 4, 300, 128
    po = rng.standard_normal((S, rows, d)).astype(np.float32)
    pl = (rng.standard_normal((S, rows)) * 5).astype(np.float32)
    pl[rng.random((S, rows)) < 0.3] = -np.inf           # empty parts
    pl[:, :3] = -np.inf                                   # rows empty everywhere
    out = torch.empty((rows, d), dtype=torch.float32, device="cuda")
    lse = torch.empty(rows, dtype=torch.float32, device="cuda")
    dpo, dpl = torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda()
    msa.msa_merge_partials(S, rows, d, dpo.data_ptr(), dpl.data_ptr(), out.data_ptr(), lse.data_ptr())
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for r in range(rows):
        want, L = O.merge_partials(list(po[:, r].astype(np.float64)), list(pl[:, r].astype(np.float64)))
        if L == -math.inf:
            assert lse[r] == -np.inf and not out[r].any()
        else:
            assert abs(lse[r] - L) <= 1e-5 * max(1.0, abs(L))
            np.testing.assert_allclose(out[r], want, rtol=0, atol=2e-6 * max(1.0, np.abs(want).max()))


def test_partial_on_a_whole_bank_equals_attend_lse():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = CASES["decode_gqa"][0]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    sh = torch.cuda.current_stream().cuda_stream
    lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
    out2, lse2 = torch.empty_like(out), torch.empty_like(lse)
    msa.msa_attend_lse(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(), lse.data_ptr(), sh)
    msa.msa_attend_partial(bank.handle, qry, w.top_k, idx.data_ptr(), 1, out2.data_ptr(), lse2.data_ptr(), sh)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    bank.close()


def test_shard_limits():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = Workload("mp_limits", 46, 1, 8, 2, 128, 12, 0, 256, 128, 64, 3, ragged=(60, 300))
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    assert msa.msa_bank_set_shard(bank.handle, -1, 20, 300, check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_bank_set_shard(bank.handle, 9, 20, 300, check=False) == msa.MSA_ERR_INVALID_ARG   # 9 + 12 > 20
    assert msa.msa_bank_set_shard(bank.handle, 0, 20, int(w.doc_lens().max()) - 1,
                                  check=False) == msa.MSA_ERR_INVALID_ARG
    bank.set_shard(8, 20, 300)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, _, _ = bank.route(qry, w.top_k, want_scores=False)
    torch.cuda.synchronize()
    ix = idx.cpu().numpy()
    assert ix.min() >= 8 and ix.max() < 20
    # the backward works on whole banks only
    out = torch.empty((1, 8, 128, 128), dtype=torch.float32, device="cuda")
    g = [torch.zeros_like(out), torch.zeros_like(LK, dtype=torch.float32), torch.zeros_like(LV, dtype=torch.float32),
         torch.zeros_like(K, dtype=torch.float32), torch.zeros_like(V, dtype=torch.float32)]
    assert msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(),
                                   *[t.data_ptr() for t in g], check=False) == msa.MSA_ERR_UNSUPPORTED
    # an index outside the whole bank raises the device flag; another shard's is skipped silently
    sel = torch.full_like(idx, 3)
    lse = torch.empty((1, 8, 128), dtype=torch.float32, device="cuda")
    assert msa.msa_attend_partial(bank.handle, qry, w.top_k, sel.data_ptr(), 0, out.data_ptr(), lse.data_ptr(),
                                  check=False) == msa.MSA_OK
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    assert torch.all(out == 0) and torch.all(torch.isinf(lse))
    sel.fill_(25)
    assert msa.msa_attend_partial(bank.handle, qry, w.top_k, sel.data_ptr(), 0, out.data_ptr(), lse.data_ptr(),
                                  check=False) == msa.MSA_OK
    assert bank.device_error() == msa.MSA_ERR_INVALID_ARG
    bank.close()
