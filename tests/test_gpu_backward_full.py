"""Full-size parity of the backward on the prefill workload (batch 1, 4096 query
tokens in 64-token routing blocks, 32/8 heads, 256 documents x 8192 tokens,
top_k 8) -- the launch bench.py --workload prefill --backward times -- on gradients
the oracle's per-row backward computes one by one:
  - dQ of sampled query rows;
  - dK and dV of every key of one selected document, summed over all the rows
    whose selection holds it (through the Parallel-RoPE adjoint);
  - dK and dV of a late local key, summed over the rows at or after it.
The upstream gradient is the bf16-exact normal tensor 77 of the workload's seed
(regenerated here from the host generator). Tolerance as in test_gpu_backward."""
import numpy as np
import pytest
import torch

import synth
from oracle import msa_oracle as O

pytestmark = pytest.mark.gpu

D_OUT_TENSOR = 77


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _close(gpu, ref, name):
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-12)
    rel_l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    worst = np.abs(gpu - ref).max() / scale
    assert rel_l2 <= 2e-2 and worst <= 4e-2, f"{name}: rel L2 {rel_l2:.2e}, max {worst:.2e} of max |ref|"


@pytest.fixture(scope="module")
def run():
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, normal, query_tensors
    w = synth.WORKLOADS["prefill"]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    torch.cuda.synchronize()
    del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    d_out = normal(tuple(out.shape), w.seed, D_OUT_TENSOR).float()
    dq = torch.empty_like(out)
    dlk = torch.empty(LK.shape, dtype=torch.float32, device="cuda")
    dlv = torch.empty(LV.shape, dtype=torch.float32, device="cuda")
    dbk = torch.zeros(K.shape, dtype=torch.float32, device="cuda")
    dbv = torch.zeros(V.shape, dtype=torch.float32, device="cuda")
    msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(), dq.data_ptr(),
                            dlk.data_ptr(), dlv.data_ptr(), dbk.data_ptr(), dbv.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    res = dict(w=w, idx=idx.cpu().numpy(), dq=dq, dlk=dlk, dlv=dlv, dbk=dbk, dbv=dbv)
    yield res
    bank.close()


class Rows:
    """The oracle's inputs for one query row, regenerated from the seeded streams."""

    def __init__(self, w, idx):
        self.w, self.idx = w, idx
        self.G, self.L, self.d, self.Lc = w.n_q_heads // w.n_kv_heads, w.doc_len, w.head_dim, w.local_len
        self.k_off = O.k_offset(w.top_k, w.doc_lens())
        self._mem, self._loc = {}, {}

    def mem(self, h, blk):
        key = (h, blk)
        if key not in self._mem:
            docs = self.idx[0, blk, h]
            L = self.L
            mk = np.concatenate([_f64(synth.bank_rows_bits(self.w, synth.T_K, h, int(j) * L, L)) for j in docs])
            mv = np.concatenate([_f64(synth.bank_rows_bits(self.w, synth.T_V, h, int(j) * L, L)) for j in docs])
            self._mem[key] = (O.parallel_rope_bank(mk, [L] * len(docs), self.w.rope_base), mv, docs)
        return self._mem[key]

    def local(self, h):
        if h not in self._loc:
            base, n = h * self.Lc * self.d, self.Lc * self.d
            self._loc[h] = (_f64(synth.normal_bf16_bits(self.w.seed, synth.T_LK, base, n)).reshape(self.Lc, self.d),
                            _f64(synth.normal_bf16_bits(self.w.seed, synth.T_LV, base, n)).reshape(self.Lc, self.d))
        return self._loc[h]

    def backward(self, hq, t):
        w, d = self.w, self.d
        h, blk = hq // self.G, t // w.route_block
        mk, mv, docs = self.mem(h, blk)
        lk, lv = self.local(h)
        off = (hq * w.q_tokens + t) * d
        q = _f64(synth.normal_bf16_bits(w.seed, synth.T_Q, off, d))
        g = _f64(synth.normal_bf16_bits(w.seed, D_OUT_TENSOR, off, d))
        return O.routed_attention_row_backward(q, self.Lc - w.q_tokens + t, self.k_off, w.rope_base, mk, mv, lk, lv, g), docs


def test_backward_full_dq_rows(run):
    w = run["w"]
    rows = Rows(w, run["idx"])
    rng = np.random.default_rng(5)
    gots, refs = [], []
    for t in [0, 63, 4095] + list(rng.integers(0, w.q_tokens, size=2)):
        hq = int(rng.integers(w.n_q_heads))
        (dq, *_), _ = rows.backward(hq, int(t))
        refs.append(dq)
        gots.append(run["dq"][0, hq, int(t)].cpu().numpy())
    _close(np.stack(gots), np.stack(refs), "dQ rows")


def test_backward_full_one_document(run):
    """dK, dV of all 8192 keys of one selected document of KV head 5."""
    w = run["w"]
    idx = run["idx"]
    h = 5
    nblk = w.q_tokens // w.route_block
    blocks_of = {}
    for blk in range(nblk):
        for j in idx[0, blk, h]:
            blocks_of.setdefault(int(j), []).append(blk)
    j = min(blocks_of, key=lambda x: (len(blocks_of[x]), x))        # the document fewest blocks selected
    rows = Rows(w, idx)
    L, G = w.doc_len, w.n_q_heads // w.n_kv_heads
    dk_rot = np.zeros((L, w.head_dim))
    dv = np.zeros((L, w.head_dim))
    for blk in blocks_of[j]:
        for g in range(G):
            for t in range(blk * w.route_block, (blk + 1) * w.route_block):
                (_, dmk, dmv, _, _), docs = rows.backward(h * G + g, t)
                pos = list(docs).index(j) * L
                dk_rot += dmk[pos:pos + L]
                dv += dmv[pos:pos + L]
    dk = O.rope_adjoint(dk_rot, np.arange(L), w.rope_base)          # back through Parallel RoPE
    r0 = h * w.kv_rows + int(np.concatenate([[0], np.cumsum(w.doc_lens())])[j])
    _close(run["dbk"][h, r0 - h * w.kv_rows:r0 - h * w.kv_rows + L].cpu().numpy(), dk, f"dK of document {j}")
    _close(run["dbv"][h, r0 - h * w.kv_rows:r0 - h * w.kv_rows + L].cpu().numpy(), dv, f"dV of document {j}")


def test_backward_full_late_local_key(run):
    """dK, dV of local key 4070 of KV head 2: the rows of tokens 4070..4095 of its 4 query heads."""
    w = run["w"]
    rows = Rows(w, run["idx"])
    h, u, G = 2, 4070, w.n_q_heads // w.n_kv_heads
    dk = np.zeros(w.head_dim)
    dv = np.zeros(w.head_dim)
    for g in range(G):
        for t in range(u - (w.local_len - w.q_tokens), w.q_tokens):
            (_, _, _, dlk, dlv), _ = rows.backward(h * G + g, t)
            dk += dlk[u]
            dv += dlv[u]
    _close(run["dlk"][0, h, u].cpu().numpy(), dk, "dK of local key 4070")
    _close(run["dlv"][0, h, u].cpu().numpy(), dv, "dV of local key 4070")
