"""Helpers of the parity tests: oracle inputs regenerated from the seeded
streams, and the comparison rules (tolerances from the routed-step contract)."""
from __future__ import annotations

import numpy as np

import synth
from oracle import msa_oracle as O

# tolerances
KR_REL = 1e-3          # pooled K_r, relative: per row (to its largest magnitude) and per element
KR_FLOOR = 1e-6        # element-wise: |gpu - ref| <= KR_REL * |ref| + KR_FLOOR (fp32 rounding of near-zero means)
SCORE_ABS = 1e-3       # router scores
TIE = 1e-3             # near-tie window for the top-k set
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
OUT_REL_L2 = 1e-2      # extra builder target (outputs are small at many keys)
OUT_MAX_ABS_F32 = 1e-4 # the fp32 path (fp32 inputs and arithmetic end to end)
ROPE_REL = 2.0 ** -8   # RoPE'd bank keys are stored in bf16


def f64(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def oracle_inputs(w: synth.Workload) -> dict:
    """Every input of a (small) workload as fp64 arrays, from the numpy generator."""
    N, Hkv, d = w.n_tokens, w.n_kv_heads, w.head_dim
    def gen(tid, shape):
        if w.dtype == "f32":
            return synth.f32_tensor(w, tid, shape).astype(np.float64)
        return synth.normal_f32(w.seed, tid, 0, int(np.prod(shape))).reshape(shape).astype(np.float64)
    if w.kv_slabs:
        def kv(tid):
            return np.stack([np.concatenate([f64(synth.doc_kv_bits(w, tid, h, j)) for j in range(w.n_docs)])
                             for h in range(Hkv)])
        K, V = kv(synth.T_K), kv(synth.T_V)
    else:
        K, V = gen(synth.T_K, (Hkv, N, d)), gen(synth.T_V, (Hkv, N, d))
    inp = {
        "K": K, "V": V,
        "R": gen(synth.T_R, (Hkv, N, w.route_dim)),
        "Q": gen(synth.T_Q, (w.batch, w.n_q_heads, w.q_tokens, d)),
        "LK": gen(synth.T_LK, (w.batch, Hkv, w.local_len, d)),
        "LV": gen(synth.T_LV, (w.batch, Hkv, w.local_len, d)),
    }
    if w.planted:
        inp["Qr"] = f64(synth.planted_qr_bits(w))
    else:
        inp["Qr"] = gen(synth.T_QR, (w.batch, Hkv, w.q_tokens, w.route_dim))
    return inp


def check_kr(gpu: np.ndarray, ref: np.ndarray):
    """K_r within 1e-3 relative: every element against its own magnitude (with a
    small absolute floor for means that sum to nearly zero), and every row against
    its largest magnitude."""
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = np.maximum(np.abs(ref).max(axis=-1, keepdims=True), 1e-30)
    err = (np.abs(gpu - ref) / scale).max()
    assert err <= KR_REL, f"K_r relative error {err:.3e}"
    bad = np.abs(gpu - ref) > KR_REL * np.abs(ref) + KR_FLOOR
    assert not bad.any(), f"{bad.sum()} K_r elements outside 1e-3 relative (+{KR_FLOOR:g})"
    return err


def check_rope_keys(gpu: np.ndarray, ref: np.ndarray):
    gpu = np.asarray(gpu, dtype=np.float64)
    bad = np.abs(gpu - ref) > ROPE_REL * np.abs(ref) + 1e-5
    assert not bad.any(), f"{bad.sum()} RoPE'd keys outside bf16 rounding"


def check_scores(gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref).max()
    assert err <= SCORE_ABS, f"router score error {err:.3e}"
    return err


def check_topk(gpu_idx: np.ndarray, gpu_top_scores: np.ndarray, gpu_scores: np.ndarray,
               ref_scores: np.ndarray, k: int):
    """gpu_idx [rows, k]; gpu_scores / ref_scores [rows, n]. Returns near-tie count.

    1. Index work is bit-exact: the selection equals a full sort of the GPU's own
       fp32 scores by (score desc, index asc).
    2. Against the oracle: the same set, except where the oracle's k-th and
       (k+1)-th scores lie within TIE; then every differing index must score
       within TIE of the oracle's k-th score.
    """
    rows, n = ref_scores.shape
    ties = 0
    for r in range(rows):
        g = gpu_scores[r].astype(np.float32)
        order = sorted(range(n), key=lambda j: (-float(g[j]), j))[:k]
        np.testing.assert_array_equal(gpu_idx[r], order, err_msg=f"row {r}: not the exact top-k of its scores")
        np.testing.assert_array_equal(gpu_top_scores[r], g[gpu_idx[r]])
        ref_sel = O.select_top_k(ref_scores[r], k)
        if set(ref_sel.tolist()) == set(gpu_idx[r].tolist()):
            continue
        s_sorted = np.sort(ref_scores[r])[::-1]
        kth = s_sorted[k - 1]
        assert k < n and kth - s_sorted[k] < TIE, f"row {r}: top-k set differs without a near tie"
        diff = set(ref_sel.tolist()) ^ set(gpu_idx[r].tolist())
        assert all(abs(ref_scores[r][j] - kth) < TIE for j in diff), f"row {r}: differing doc not near the tie"
        ties += 1
    return ties


def check_out(gpu: np.ndarray, ref: np.ndarray, max_abs: float = OUT_MAX_ABS):
    gpu = np.asarray(gpu, dtype=np.float64)
    d = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    assert d.max() <= max_abs, f"max-abs {d.max():.3e} (bound {max_abs:g})"
    assert d.mean() <= OUT_MEAN_ABS, f"mean-abs {d.mean():.3e}"
    assert rel <= OUT_REL_L2, f"relative L2 {rel:.3e}"
    return d.max(), d.mean(), rel
