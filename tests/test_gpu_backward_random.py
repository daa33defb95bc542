"""Randomised shape sweep of the backward: seeded small workloads, half of them on
the shapes of the tensor-core backward (head_dim 128, 64- or 128-token routing
blocks), the rest anywhere (head_dim 64 or 128, any block size, ragged documents
and local tails), every gradient compared with the oracle's backward over the
GPU's own selection. Even cases call msa_attend_backward (which recomputes the
forward's state), odd ones msa_attend_lse then msa_attend_backward_saved.
Tolerance as in test_gpu_backward."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P

pytestmark = pytest.mark.gpu

D_OUT_TENSOR = 79


def _case(i: int) -> Workload:
    rng = np.random.RandomState(9100 + i)
    tc = i % 2 == 0
    while True:
        d = 128 if tc else int(rng.choice([64, 128]))
        hkv = int(rng.choice([1, 2, 4]))
        g = int(rng.choice([1, 2, 4, 8]))
        bq = int(rng.choice([64, 128])) if tc else int(rng.choice([1, 2, 3, 4, 8, 16, 32, 48]))
        nblk = int(rng.randint(1, 3)) if bq >= 32 else int(rng.randint(1, 9))
        tq = bq * nblk
        lc = tq + int(rng.randint(0, 200))
        b = int(rng.randint(1, 3))
        n_docs = int(rng.randint(2, 25))
        lo = int(rng.randint(1, 150))
        hi = int(rng.randint(lo + 1, 700))
        top_k = int(rng.randint(1, min(n_docs, 12) + 1))
        rows = b * hkv * g * tq
        keys = top_k * (lo + hi) / 2 + lc
        if rows * keys <= 1.2e6:
            return Workload(f"bwd_rand{i}", 9100 + i, b, hkv * g, hkv, d, n_docs, 0, lc, tq, bq, top_k,
                            ragged=(lo, hi))


CASES = [_case(i) for i in range(16)]


def _close(gpu, ref, name):
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-12)
    rel_l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    worst = np.abs(gpu - ref).max() / scale
    assert rel_l2 <= 2e-2 and worst <= 4e-2, f"{name}: rel L2 {rel_l2:.2e}, max {worst:.2e} of max |ref|"


@pytest.mark.parametrize("i", range(len(CASES)), ids=[c.name for c in CASES])
def test_random_shape_backward(i):
    import sparse_attention_routed_b200 as msa
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, normal, query_tensors
    w = CASES[i]
    K, V, R = bank_tensors(w)
    Q, Qr, LK, LV = query_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    s = torch.cuda.current_stream().cuda_stream
    d_out = normal(tuple(out.shape), w.seed, D_OUT_TENSOR).float()
    g = [torch.empty_like(out), torch.empty(LK.shape, dtype=torch.float32, device="cuda"),
         torch.empty(LV.shape, dtype=torch.float32, device="cuda"),
         torch.zeros(K.shape, dtype=torch.float32, device="cuda"),
         torch.zeros(V.shape, dtype=torch.float32, device="cuda")]
    if i % 2 == 0:
        msa.msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(),
                                *[x.data_ptr() for x in g], s)
    else:
        out2 = torch.empty_like(out)
        lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
        msa.msa_attend_lse(bank.handle, qry, w.top_k, idx.data_ptr(), out2.data_ptr(), lse.data_ptr(), s)
        msa.msa_attend_backward_saved(bank.handle, qry, w.top_k, idx.data_ptr(), out2.data_ptr(), lse.data_ptr(),
                                      d_out.data_ptr(), *[x.data_ptr() for x in g], s)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    inp = P.oracle_inputs(w)
    ref = O.backward(inp, w.doc_lens(), w.top_k, w.route_block, d_out.cpu().numpy().astype(np.float64),
                     w.rope_base, selection=idx.cpu().numpy())
    for x, key in zip(g, ["dQ", "dLK", "dLV", "dK", "dV"]):
        _close(x.cpu().numpy(), ref[key], f"{w.name} {key}")
    bank.close()
