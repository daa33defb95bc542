"""Full-size parity on the prefill workload (batch 1, 4096 query tokens in 64-token
routing blocks, 32/8 heads, 256 documents x 8192 tokens, top_k 8), on outputs the
oracle computes one by one: every document score and the top-8 of all 64 routing
blocks for one KV head, and 8 random output rows over the GPU's selection."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.fixture(scope="module")
def run():
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors
    w = synth.WORKLOADS["prefill"]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    torch.cuda.synchronize()
    del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, tsc, scores = bank.route(qry, w.top_k)
    out = bank.attend(qry, w.top_k, idx)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = dict(w=w, idx=idx.cpu().numpy(), tsc=tsc.cpu().numpy(), scores=scores.cpu().numpy(),
               out=out.cpu().numpy())
    bank.close()
    return res


def test_prefill_router_one_head(run):
    w = run["w"]
    h, n, L = 3, w.n_docs, w.doc_len
    kr = np.empty((n * (L // 256), w.route_dim))
    for j in range(n):
        kr[j * (L // 256):(j + 1) * (L // 256)] = O.chunk_mean_pool(
            _f64(synth.bank_rows_bits(w, synth.T_R, h, j * L, L)))
    chunk_doc = np.repeat(np.arange(n), L // 256)
    Qr = _f64(synth.query_bits(w, synth.T_QR, (w.batch, w.n_kv_heads, w.q_tokens, w.route_dim)))
    qb = O.block_mean_query(Qr[0, h], w.route_block)
    ref = np.stack([O.doc_max(O.chunk_cosines(qb[blk], kr), chunk_doc, n) for blk in range(qb.shape[0])])
    gpu = run["scores"][0, :, h, :]
    P.check_scores(gpu, ref)
    P.check_topk(run["idx"][0, :, h, :], run["tsc"][0, :, h, :], gpu, ref, w.top_k)


def test_prefill_sampled_rows(run):
    w = run["w"]
    rng = np.random.default_rng(3)
    G, L, d, Lc = w.n_q_heads // w.n_kv_heads, w.doc_len, w.head_dim, w.local_len
    k_off = O.k_offset(w.top_k, w.doc_lens())
    gots, refs = [], []
    for t in [0, 63, 64, 2000, 4095] + list(rng.integers(0, w.q_tokens, size=3)):
        hq = int(rng.integers(w.n_q_heads))
        h, blk = hq // G, int(t) // w.route_block
        docs = run["idx"][0, blk, h]
        mk = np.concatenate([_f64(synth.bank_rows_bits(w, synth.T_K, h, int(j) * L, L)) for j in docs])
        mv = np.concatenate([_f64(synth.bank_rows_bits(w, synth.T_V, h, int(j) * L, L)) for j in docs])
        base = h * Lc * d
        lk = _f64(synth.normal_bf16_bits(w.seed, synth.T_LK, base, Lc * d)).reshape(Lc, d)
        lv = _f64(synth.normal_bf16_bits(w.seed, synth.T_LV, base, Lc * d)).reshape(Lc, d)
        q = _f64(synth.normal_bf16_bits(w.seed, synth.T_Q, (hq * w.q_tokens + int(t)) * d, d))
        mk_rot = O.parallel_rope_bank(mk, [L] * len(docs), w.rope_base)
        refs.append(O.routed_attention_row(q, Lc - w.q_tokens + int(t), k_off, w.rope_base, mk_rot, mv, lk, lv))
        gots.append(run["out"][0, hq, int(t)])
    P.check_out(np.stack(gots), np.stack(refs))
