"""Full-size parity on the benchmark workload (decode_4m: 4.19M-token bank,
batch 8, 32/8 heads, top_k 16), on outputs the oracle computes one by one, through
msa_route then msa_attend; the launch configuration bench.py times (msa_forward:
programmatic dependent launches, the local context's CTAs beside the router) must
give the same selection and output bit for bit:

* K_r of 256 random (head, chunk) pairs and the RoPE'd keys of 256 random tokens;
* every document score and the top-16 of all 8 sequences for one KV head
  (the oracle pools that head's whole bank: 16384 chunks);
* the attention output of all 256 (sequence, query head) rows over the GPU's
  selection (checked above to be a correct top-k).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def run():
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = synth.WORKLOADS["decode_4m"]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    torch.cuda.synchronize()
    del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    bank.reserve(qry, w.top_k)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    idx_f, out_f = bank.forward(qry, w.top_k)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = dict(w=w, bank=bank, K=K, idx=idx.cpu().numpy(), tsc=tsc.cpu().numpy(),
               scores=scores.cpu().numpy(), out=out.cpu().numpy(), kr=bank.k_r(),
               idx_f=idx_f.cpu().numpy(), out_f=out_f.cpu().numpy())
    yield res
    bank.close()


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def test_sampled_pooling_and_rope(run):
    w, kr = run["w"], run["kr"]
    rng = np.random.default_rng(7)
    L, d = w.doc_len, w.head_dim
    for _ in range(256):
        h, c = int(rng.integers(w.n_kv_heads)), int(rng.integers(kr.shape[1]))
        rows = _f64(synth.bank_rows_bits(w, synth.T_R, h, c * 256, 256))
        P.check_kr(kr[h, c:c + 1].cpu().numpy(), O.chunk_mean_pool(rows))
    toks = rng.integers(0, w.n_tokens, size=256)
    heads = rng.integers(0, w.n_kv_heads, size=256)
    gpu = run["K"][torch.as_tensor(heads, device="cuda"), torch.as_tensor(toks, device="cuda")].float().cpu().numpy()
    for i, (h, t) in enumerate(zip(heads, toks)):
        raw = _f64(synth.bank_rows_bits(w, synth.T_K, int(h), int(t), 1))[0]
        P.check_rope_keys(gpu[i], O.rope(raw, int(t) % L, w.rope_base))


def test_full_router_one_head(run):
    w = run["w"]
    h = 5
    n, L = w.n_docs, w.doc_len
    kr = np.empty((n * (L // 256), w.route_dim))
    for j in range(n):
        kr[j * (L // 256):(j + 1) * (L // 256)] = O.chunk_mean_pool(
            _f64(synth.bank_rows_bits(w, synth.T_R, h, j * L, L)))
    chunk_doc = np.repeat(np.arange(n), L // 256)
    Qr = _f64(synth.query_bits(w, synth.T_QR, (w.batch, w.n_kv_heads, 1, w.route_dim)))
    ref = np.stack([O.doc_max(O.chunk_cosines(Qr[b, h, 0], kr), chunk_doc, n) for b in range(w.batch)])
    gpu = run["scores"][:, 0, h, :]
    P.check_scores(gpu, ref)
    P.check_topk(run["idx"][:, 0, h, :], run["tsc"][:, 0, h, :], gpu, ref, w.top_k)


def test_all_attention_rows(run):
    """Every output row of the step (8 sequences x 32 query heads), each against the
    oracle's attention over the GPU's own selection (16 documents + 4096 local keys)."""
    w = run["w"]
    G, L, d, Lc = w.n_q_heads // w.n_kv_heads, w.doc_len, w.head_dim, w.local_len
    k_off = O.k_offset(w.top_k, w.doc_lens())
    Q = _f64(synth.query_bits(w, synth.T_Q, (w.batch, w.n_q_heads, 1, d)))
    gots, refs = [], []
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            docs = run["idx"][b, 0, h]
            mk = np.concatenate([_f64(synth.bank_rows_bits(w, synth.T_K, h, int(j) * L, L)) for j in docs])
            mv = np.concatenate([_f64(synth.bank_rows_bits(w, synth.T_V, h, int(j) * L, L)) for j in docs])
            base = (b * w.n_kv_heads + h) * Lc * d
            lk = _f64(synth.normal_bf16_bits(w.seed, synth.T_LK, base, Lc * d)).reshape(Lc, d)
            lv = _f64(synth.normal_bf16_bits(w.seed, synth.T_LV, base, Lc * d)).reshape(Lc, d)
            mk_rot = O.parallel_rope_bank(mk, [L] * len(docs), w.rope_base)
            for hq in range(h * G, (h + 1) * G):
                refs.append(O.routed_attention_row(Q[b, hq, 0], Lc - 1, k_off, w.rope_base, mk_rot, mv, lk, lv))
                gots.append(run["out"][b, hq, 0])
    assert len(gots) == w.batch * w.n_q_heads
    P.check_out(np.stack(gots), np.stack(refs))


def test_forward_equals_route_then_attend(run):
    """msa_forward, as bench.py times it, gives the bits of msa_route + msa_attend."""
    np.testing.assert_array_equal(run["idx_f"], run["idx"])
    np.testing.assert_array_equal(run["out_f"], run["out"])
