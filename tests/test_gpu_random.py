"""Randomised shape sweep: seeded small workloads that together reach every
kernel path (decode, mma.sync prefill and tcgen05 prefill attention; mma.sync
and tcgen05 routers; fused and separate q_r), each compared with the oracle
element by element exactly as in test_gpu_parity."""
import numpy as np
import pytest

from oracle import msa_oracle as O
from synth import Workload
from tests import parity as P
from tests.test_gpu_parity import run_gpu

pytestmark = pytest.mark.gpu


def _case(i: int) -> Workload:
    rng = np.random.RandomState(7000 + i)
    while True:
        d = int(rng.choice([64, 128]))
        hkv = int(rng.choice([1, 2, 4]))
        g = int(rng.choice([1, 2, 4, 8]))
        bq = int(rng.choice([1, 2, 3, 4, 8, 16, 32, 64, 128]))
        nblk = int(rng.randint(1, 4)) if bq >= 16 else int(rng.randint(1, 13))
        tq = bq * nblk
        lc = tq + int(rng.randint(0, 300))
        b = int(rng.randint(1, 4))
        n_docs = int(rng.randint(3, 41))
        lo = int(rng.randint(1, 100))
        hi = int(rng.randint(lo + 1, 1200))
        top_k = int(rng.randint(1, min(n_docs, 64) + 1))
        rows = b * hkv * g * tq
        keys = top_k * (lo + hi) / 2 + lc
        if rows * keys <= 2.5e6 and b * nblk * hkv <= 65535:
            return Workload(f"rand{i}", 7000 + i, b, hkv * g, hkv, d, n_docs, 0, lc, tq, bq, top_k, ragged=(lo, hi))


CASES = [_case(i) for i in range(24)]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_random_shape_parity(w):
    g = run_gpu(w)
    inp = P.oracle_inputs(w)
    ref = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base)
    P.check_kr(g["K_r"], ref["K_r"])
    P.check_rope_keys(g["K_rot"], ref["K_rot"])
    rows = g["scores"].reshape(-1, w.n_docs)
    P.check_scores(rows, ref["doc_scores"].reshape(-1, w.n_docs))
    P.check_topk(g["idx"].reshape(-1, w.top_k), g["tsc"].reshape(-1, w.top_k), rows,
                 ref["doc_scores"].reshape(-1, w.n_docs), w.top_k)
    ref2 = O.forward(inp, w.doc_lens(), w.top_k, w.route_block, w.rope_base, selection=g["idx"])
    P.check_out(g["out"], ref2["out"])
    np.testing.assert_array_equal(g["idx2"], g["idx"])
    np.testing.assert_array_equal(g["out2"], g["out"])
