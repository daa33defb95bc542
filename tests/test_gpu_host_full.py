"""Full-size parity of the pinned-host tier on the bank_100m workload (24414 documents
x 4096 tokens = 100M tokens, K/V in pinned host memory over 1024 slabs, 16 decode
sequences, 32/8 heads, top_k 16) and the ragged_planted workload (8192 documents of
512-16384 tokens = 69M tokens, 4 sequences, 64/8 heads, top_k 32, planted routing
queries) -- the launches bench.py --workload bank_100m / ragged_planted time -- on
outputs the oracle computes one by one:
  - the top-k of every (sequence, KV head) row is exactly the top-k of the GPU's own
    scores (index work, every document of the bank);
  - for one row, the oracle's scores of the selected documents and of 48 random other
    documents (pooling their routing keys afresh) match the GPU's, and no sampled
    unselected document beats a selected one by more than the near-tie window;
  - sampled output rows of msa_forward over the GPU's selection (the selected
    documents' K/V regenerated through the slab mapping)."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.fixture(scope="module", params=["bank_100m", "ragged_planted"])
def run(request):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import fill_normal, host_kv_pool, query_tensors
    w = synth.WORKLOADS[request.param]
    Hkv, d, B, k = w.n_kv_heads, w.head_dim, w.batch, w.top_k
    Kh, Vh = host_kv_pool(w)
    bank = Bank(Kh, Vh, w.doc_lens(), w.rope_base, kv_location=msa.MSA_KV_PINNED_HOST, doc_rows=w.doc_kv_rows())
    off = np.concatenate([[0], np.cumsum(w.doc_lens())])
    for j0 in range(0, w.n_docs, 64):          # routing keys streamed through the build, as bench.py does
        j1 = min(w.n_docs, j0 + 64)
        T = int(off[j1] - off[j0])
        R = torch.empty((Hkv, T, d), dtype=torch.bfloat16, device="cuda")
        for h in range(Hkv):
            fill_normal(R[h], w.seed, synth.T_R, (h * w.n_tokens + int(off[j0])) * d)
        bank.build(R, j0, j1, rope=False)
        del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx = torch.empty((B, 1, Hkv, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.n_q_heads, 1, d), dtype=torch.float32, device="cuda")
    scores = torch.empty((B, 1, Hkv, w.n_docs), dtype=torch.float32, device="cuda")
    tsc = torch.empty((B, 1, Hkv, k), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    msa.msa_forward(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), s)
    idx2 = torch.empty_like(idx)
    msa.msa_route(bank.handle, qry, k, scores.data_ptr(), idx2.data_ptr(), tsc.data_ptr(), s)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = dict(w=w, idx=idx.cpu().numpy(), idx2=idx2.cpu().numpy(), scores=scores.cpu().numpy(),
               tsc=tsc.cpu().numpy(), out=out.cpu().numpy(), off=off)
    bank.close()
    del Kh, Vh
    return res


def test_host_full_topk_exact_on_own_scores(run):
    w = run["w"]
    np.testing.assert_array_equal(run["idx2"], run["idx"])      # msa_forward routes as msa_route does
    rows = run["scores"].reshape(-1, w.n_docs)
    sel = run["idx"].reshape(-1, w.top_k)
    for r in range(rows.shape[0]):
        g = rows[r].astype(np.float32)
        order = np.lexsort((np.arange(w.n_docs), -g.astype(np.float64)))[:w.top_k]
        np.testing.assert_array_equal(sel[r], order, err_msg=f"row {r}")
        np.testing.assert_array_equal(run["tsc"].reshape(-1, w.top_k)[r], g[sel[r]])


def test_host_full_router_sample(run):
    w = run["w"]
    b, h = w.batch - 1, 6
    rng = np.random.default_rng(7)
    sel = [int(j) for j in run["idx"][b, 0, h]]
    others = [int(j) for j in rng.choice(np.setdiff1d(np.arange(w.n_docs), sel), size=48, replace=False)]
    if w.planted:
        Qr = _f64(synth.planted_qr_bits(w))
    else:
        Qr = _f64(synth.query_bits(w, synth.T_QR, (w.batch, w.n_kv_heads, w.q_tokens, w.route_dim)))
    q = O.block_mean_query(Qr[b, h], w.route_block)[0]
    off = run["off"]
    ref = {}
    for j in sel + others:
        Rj = _f64(synth.bank_rows_bits(w, synth.T_R, h, int(off[j]), int(off[j + 1] - off[j])))
        ref[j] = O.doc_max(O.chunk_cosines(q, O.chunk_mean_pool(Rj)), np.zeros(len(O.chunk_spans(len(Rj))), int), 1)[0]
    got = run["scores"][b, 0, h]
    P.check_scores(np.array([got[j] for j in ref]), np.array([ref[j] for j in ref]))
    kth = min(ref[j] for j in sel)
    assert all(ref[j] <= kth + P.TIE for j in others), "an unselected sampled document beats a selected one"


def test_host_full_output_rows(run):
    w = run["w"]
    rng = np.random.default_rng(8)
    G, d, Lc = w.n_q_heads // w.n_kv_heads, w.head_dim, w.local_len
    k_off = O.k_offset(w.top_k, w.doc_lens())
    gots, refs = [], []
    for _ in range(6):
        b, hq = int(rng.integers(w.batch)), int(rng.integers(w.n_q_heads))
        h = hq // G
        docs = [int(j) for j in run["idx"][b, 0, h]]
        lens = [int(w.doc_lens()[j]) for j in docs]
        mk = np.concatenate([_f64(synth.doc_kv_bits(w, synth.T_K, h, j)) for j in docs])
        mv = np.concatenate([_f64(synth.doc_kv_bits(w, synth.T_V, h, j)) for j in docs])
        base = (b * w.n_kv_heads + h) * Lc * d
        lk = _f64(synth.normal_bf16_bits(w.seed, synth.T_LK, base, Lc * d)).reshape(Lc, d)
        lv = _f64(synth.normal_bf16_bits(w.seed, synth.T_LV, base, Lc * d)).reshape(Lc, d)
        q = _f64(synth.normal_bf16_bits(w.seed, synth.T_Q, ((b * w.n_q_heads + hq) * w.q_tokens) * d, d))
        mk_rot = O.parallel_rope_bank(mk, lens, w.rope_base)
        refs.append(O.routed_attention_row(q, Lc - w.q_tokens, k_off, w.rope_base, mk_rot, mv, lk, lv))
        gots.append(run["out"][b, hq, 0])
    P.check_out(np.stack(gots), np.stack(refs))
