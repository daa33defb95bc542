"""The document selection on its own (the msa_selftest_topk hook of the C ABI):
both top-k kernels, the block-per-row radix select and the warp-per-row select,
against a host ranking of the same fp32 scores by (score descending, index
ascending), bit for bit, and against each other.

Scores compare through the IEEE total order of their bits, as the hook documents;
the cases hold ties (integer-valued scores, all equal), infinities, a lane of the
warp kernel that holds every winner (so that more than 64 keys pass its threshold
and it takes its extract-the-maximum path), short rows and row counts that leave a
CTA of the warp kernel partly empty."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _order_keys(s: np.ndarray) -> np.ndarray:
    b = s.astype(np.float32).view(np.uint32).astype(np.uint64)
    neg = (b & 0x80000000) != 0
    return np.where(neg, (~b) & 0xFFFFFFFF, b | 0x80000000)


def _host_topk(scores: np.ndarray, k: int) -> np.ndarray:
    rows, n = scores.shape
    out = np.empty((rows, k), np.int64)
    for r in range(rows):
        key = _order_keys(scores[r])
        out[r] = np.lexsort((np.arange(n), -key.astype(np.float64)))[:k]
    return out


def _scores(kind: str, rows: int, n: int, rng) -> np.ndarray:
    if kind == "normal":
        return rng.standard_normal((rows, n)).astype(np.float32)
    if kind == "ties":
        return rng.integers(-3, 4, (rows, n)).astype(np.float32)
    if kind == "equal":
        return np.full((rows, n), 0.25, np.float32)
    if kind == "hot_lane":  # every large score in lane 5 of the warp kernel (indices 5 mod 32)
        s = rng.standard_normal((rows, n)).astype(np.float32) - 10.0
        s[:, 5::32] += 20.0
        return s
    if kind == "inf":
        s = rng.uniform(-1, 1, (rows, n)).astype(np.float32)
        s[:, rng.integers(0, n, 3)] = np.inf
        s[:, rng.integers(0, n, 3)] = -np.inf
        return s
    raise ValueError(kind)


def _run(scores: np.ndarray, k: int, path: int):
    from sparse_attention_routed_b200 import msa_selftest_topk
    rows, n = scores.shape
    d = torch.from_numpy(scores).cuda()
    idx = torch.full((rows, k), -1, dtype=torch.int32, device="cuda")
    top = torch.full((rows, k), np.nan, dtype=torch.float32, device="cuda")
    msa_selftest_topk(d.data_ptr(), rows, n, k, idx.data_ptr(), top.data_ptr(), path,
                      torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), top.cpu().numpy()


CASES = [(n, k) for n in (1, 7, 32, 33, 255, 256, 300, 1000, 1024, 1500, 2048) for k in (1, 8, 16, 32) if k <= n]


@pytest.mark.parametrize("kind", ["normal", "ties", "equal", "hot_lane", "inf"])
def test_both_kernels_match_host_ranking(kind):
    rng = np.random.default_rng(11)
    for n, k in CASES:
        rows = 7 if n > 1000 else 9
        s = _scores(kind, rows, n, rng)
        ref = _host_topk(s, k)
        for path in (1, 2):
            idx, top = _run(s, k, path)
            np.testing.assert_array_equal(idx, ref, err_msg=f"{kind} n={n} k={k} path={path}")
            np.testing.assert_array_equal(top.view(np.uint32), np.take_along_axis(s, ref, 1).view(np.uint32))


def test_block_kernel_large_rows_and_k():
    """Shapes only the radix select takes: n above 2048 and k above 32."""
    rng = np.random.default_rng(12)
    for n, k, kind in ((5000, 32, "normal"), (24414, 16, "normal"), (8192, 64, "ties"), (40, 33, "ties"),
                       (3000, 64, "hot_lane")):
        s = _scores(kind, 3, n, rng)
        idx, top = _run(s, k, 1)
        np.testing.assert_array_equal(idx, _host_topk(s, k), err_msg=f"n={n} k={k}")
        auto, _ = _run(s, k, 0)
        np.testing.assert_array_equal(auto, idx)


def test_warp_kernel_limits():
    from sparse_attention_routed_b200 import MSA_ERR_INVALID_ARG, msa_selftest_topk
    s = torch.zeros((2, 4096), dtype=torch.float32, device="cuda")
    idx = torch.empty((2, 64), dtype=torch.int32, device="cuda")
    assert msa_selftest_topk(s.data_ptr(), 2, 4096, 8, idx.data_ptr(), 0, 2, check=False) == MSA_ERR_INVALID_ARG
    assert msa_selftest_topk(s.data_ptr(), 2, 2048, 33, idx.data_ptr(), 0, 2, check=False) == MSA_ERR_INVALID_ARG
    assert msa_selftest_topk(s.data_ptr(), 2, 16, 17, idx.data_ptr(), 0, 1, check=False) == MSA_ERR_INVALID_ARG
    assert msa_selftest_topk(s.data_ptr(), 2, 2048, 65, idx.data_ptr(), 0, 1, check=False) == MSA_ERR_INVALID_ARG
    assert msa_selftest_topk(s.data_ptr(), 2, 2048, 8, idx.data_ptr(), 0, 3, check=False) == MSA_ERR_INVALID_ARG
