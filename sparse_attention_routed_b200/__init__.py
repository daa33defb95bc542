"""Python binding of libmsa (routed sparse attention of Memory Sparse Attention on B200).

Argument marshalling only: every step runs in the CUDA library. The functions
carry the names of the C entry points in include/msa.h and take raw integers
(device pointers, host arrays via numpy, stream handles). `ptr()` turns a
torch tensor into its device pointer after checking dtype and contiguity.

The first call loads libmsa.so (lib()) and fails loudly when it is missing or
lacks an entry point; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_OK = 0
MSA_ERR_INVALID_ARG = 1
MSA_ERR_UNSUPPORTED = 2
MSA_ERR_OOM = 3
MSA_ERR_CUDA = 4
MSA_ERR_TIMEOUT = 5
MSA_ERR_HOST_TIER = 6

MSA_KV_DEVICE = 0
MSA_KV_PINNED_HOST = 1
MSA_KR_F32 = 0
MSA_KR_BF16 = 1
MSA_FETCH_COPY_ENGINE = 0
MSA_FETCH_SM_GATHER = 1
MSA_DTYPE_BF16 = 0
MSA_DTYPE_F32 = 1


class MsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {msa_status_string(status)} (status {status})")
        self.status = status


class msa_bank_config(ctypes.Structure):
    _fields_ = [
        ("n_docs", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("route_dim", ctypes.c_int32), ("doc_lens", ctypes.POINTER(ctypes.c_int64)),
        ("rope_base", ctypes.c_float), ("kv_location", ctypes.c_int32), ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p), ("kv_rows", ctypes.c_int64), ("doc_rows", ctypes.POINTER(ctypes.c_int64)),
        ("dtype", ctypes.c_int32),
    ]


class msa_query(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("q_tokens", ctypes.c_int32),
        ("local_len", ctypes.c_int32), ("route_block", ctypes.c_int32), ("q", ctypes.c_void_p),
        ("qr", ctypes.c_void_p), ("local_k", ctypes.c_void_p), ("local_v", ctypes.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmsa.so is not built ({LIB_PATH}); run python -m sparse_attention_routed_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "msa_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "msa_bank_create": ([ctypes.POINTER(msa_bank_config), ctypes.POINTER(vp)], ctypes.c_int),
        "msa_bank_destroy": ([vp], ctypes.c_int),
        "msa_build_bank": ([vp, i32, i32, vp, i64, vp, i64, vp], ctypes.c_int),
        "msa_bank_info": ([vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i64),
                           ctypes.POINTER(vp), ctypes.POINTER(vp)], ctypes.c_int),
        "msa_reserve": ([vp, ctypes.POINTER(msa_query), i32], ctypes.c_int),
        "msa_route": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp, vp], ctypes.c_int),
        "msa_attend": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp], ctypes.c_int),
        "msa_forward": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp], ctypes.c_int),
        "msa_get_device_error": ([vp, vp], ctypes.c_int),
        "msa_route_noalloc": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp, vp], ctypes.c_int),
        "msa_attend_lse": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp, vp], ctypes.c_int),
        "msa_attend_backward": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "msa_attend_backward_saved": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
                                      ctypes.c_int),
        "msa_set_kv_cache": ([vp, i64], ctypes.c_int),
        "msa_kv_cache_stats": ([vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i64)], ctypes.c_int),
        "msa_set_host_fetch": ([vp, ctypes.c_int], ctypes.c_int),
        "msa_get_host_fetch": ([vp, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
        "msa_set_router_precision": ([vp, ctypes.c_int], ctypes.c_int),
        "msa_check_wait_timeout": ([vp, vp], ctypes.c_int),
        "msa_selftest_exp2_poly": ([vp, vp, vp, i64, vp], ctypes.c_int),
        "msa_selftest_topk": ([vp, i32, i32, i32, vp, vp, i32, vp], ctypes.c_int),
        "msa_bank_set_shard": ([vp, i32, i32, i64], ctypes.c_int),
        "msa_attend_partial": ([vp, ctypes.POINTER(msa_query), i32, vp, i32, vp, vp, vp], ctypes.c_int),
        "msa_merge_topk": ([i32, i32, i32, vp, vp, vp, vp, vp], ctypes.c_int),
        "msa_merge_partials": ([i32, i64, i32, vp, vp, vp, vp, vp], ctypes.c_int),
        "msa_interleave_route": ([vp, ctypes.POINTER(msa_query), i32, vp, vp, i32, vp, vp, vp, vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_LIB = None


def lib():
    """The loaded libmsa.so (loaded on first use)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "LIB":
        return lib()
    raise AttributeError(name)

# Every symbol include/msa.h and include/msa_selftest.h declare, in declaration order.
EXPORTED = ["msa_bank_create", "msa_bank_destroy", "msa_build_bank", "msa_bank_info", "msa_reserve",
            "msa_route", "msa_attend", "msa_attend_lse", "msa_attend_backward", "msa_attend_backward_saved",
            "msa_forward", "msa_route_noalloc", "msa_bank_set_shard", "msa_attend_partial", "msa_merge_topk",
            "msa_merge_partials", "msa_interleave_route", "msa_set_kv_cache",
            "msa_kv_cache_stats", "msa_set_host_fetch", "msa_get_host_fetch", "msa_set_router_precision", "msa_check_wait_timeout", "msa_get_device_error",
            "msa_status_string", "msa_selftest_exp2_poly", "msa_selftest_topk"]


def msa_status_string(status: int) -> str:
    return lib().msa_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MSA_OK:
        raise MsaError(status, where)


def ptr(t, dtype=None) -> int:
    """Device (or pinned host) pointer of a contiguous torch tensor; 0 for None."""
    if t is None:
        return 0
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def make_query(batch, n_q_heads, q_tokens, local_len, route_block, q=0, qr=0, local_k=0, local_v=0) -> msa_query:
    return msa_query(batch, n_q_heads, q_tokens, local_len, route_block, q or None, qr or None,
                     local_k or None, local_v or None)


def msa_bank_create(n_docs: int, n_kv_heads: int, head_dim: int, doc_lens, k: int, v: int,
                    rope_base: float = 10000.0, kv_location: int = MSA_KV_DEVICE, kv_rows: int = 0,
                    doc_rows=None, route_dim: Optional[int] = None, check: bool = True,
                    dtype: int = MSA_DTYPE_BF16):
    """Returns (status, handle). doc_lens / doc_rows are host int64 sequences."""
    lens = np.ascontiguousarray(np.asarray(doc_lens, dtype=np.int64))
    rows = None if doc_rows is None else np.ascontiguousarray(np.asarray(doc_rows, dtype=np.int64))
    cfg = msa_bank_config(
        n_docs, n_kv_heads, head_dim, head_dim if route_dim is None else route_dim,
        lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), rope_base, kv_location, k or None, v or None,
        kv_rows, None if rows is None else rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), dtype)
    handle = ctypes.c_void_p()
    st = lib().msa_bank_create(ctypes.byref(cfg), ctypes.byref(handle))
    if check:
        _check(st, "msa_bank_create")
    return st, handle.value


def msa_bank_destroy(bank) -> int:
    return lib().msa_bank_destroy(bank)


def msa_build_bank(bank, doc_begin, doc_end, r_slice, r_head_stride, k_slice, k_head_stride, stream=0,
                   check=True) -> int:
    st = lib().msa_build_bank(bank, doc_begin, doc_end, r_slice or None, r_head_stride, k_slice or None,
                            k_head_stride, stream or None)
    if check:
        _check(st, "msa_build_bank")
    return st


def msa_bank_info(bank):
    n_tok, n_ch, max_len = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    kr, kinv = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib().msa_bank_info(bank, ctypes.byref(n_tok), ctypes.byref(n_ch), ctypes.byref(max_len),
                             ctypes.byref(kr), ctypes.byref(kinv)), "msa_bank_info")
    return {"n_tokens": n_tok.value, "n_chunks": n_ch.value, "max_doc_len": max_len.value,
            "k_r": kr.value, "k_r_inv_norm": kinv.value}


def msa_reserve(bank, query: msa_query, top_k: int, check=True) -> int:
    st = lib().msa_reserve(bank, ctypes.byref(query), top_k)
    if check:
        _check(st, "msa_reserve")
    return st


def msa_route(bank, query: msa_query, top_k: int, doc_scores: int, topk_idx: int, topk_scores: int,
              stream=0, check=True) -> int:
    st = lib().msa_route(bank, ctypes.byref(query), top_k, doc_scores or None, topk_idx or None,
                       topk_scores or None, stream or None)
    if check:
        _check(st, "msa_route")
    return st


def msa_attend(bank, query: msa_query, top_k: int, topk_idx: int, out: int, stream=0, check=True) -> int:
    st = lib().msa_attend(bank, ctypes.byref(query), top_k, topk_idx or None, out or None, stream or None)
    if check:
        _check(st, "msa_attend")
    return st


def msa_attend_lse(bank, query: msa_query, top_k: int, topk_idx: int, out: int, lse: int, stream=0,
                   check=True) -> int:
    st = lib().msa_attend_lse(bank, ctypes.byref(query), top_k, topk_idx or None, out or None, lse or None,
                              stream or None)
    if check:
        _check(st, "msa_attend_lse")
    return st


def msa_forward(bank, query: msa_query, top_k: int, topk_idx: int, out: int, stream=0, check=True) -> int:
    st = lib().msa_forward(bank, ctypes.byref(query), top_k, topk_idx or None, out or None, stream or None)
    if check:
        _check(st, "msa_forward")
    return st


def msa_route_noalloc(bank, query: msa_query, top_k: int, doc_scores: int, topk_idx: int, topk_scores: int,
                      stream=0, check=True) -> int:
    """msa_route with its scratch in the library's fixed 4 MiB device array (no allocation)."""
    st = lib().msa_route_noalloc(bank, ctypes.byref(query), top_k, doc_scores or None, topk_idx or None,
                               topk_scores or None, stream or None)
    if check:
        _check(st, "msa_route_noalloc")
    return st


def msa_attend_backward(bank, query: msa_query, top_k: int, topk_idx: int, d_out: int, dq: int, dlocal_k: int,
                        dlocal_v: int, dbank_k: int, dbank_v: int, stream=0, check=True) -> int:
    st = lib().msa_attend_backward(bank, ctypes.byref(query), top_k, topk_idx or None, d_out or None, dq or None,
                                   dlocal_k or None, dlocal_v or None, dbank_k or None, dbank_v or None,
                                   stream or None)
    if check:
        _check(st, "msa_attend_backward")
    return st


def msa_attend_backward_saved(bank, query: msa_query, top_k: int, topk_idx: int, out: int, lse: int, d_out: int,
                              dq: int, dlocal_k: int, dlocal_v: int, dbank_k: int, dbank_v: int, stream=0,
                              check=True) -> int:
    st = lib().msa_attend_backward_saved(bank, ctypes.byref(query), top_k, topk_idx or None, out or None,
                                         lse or None, d_out or None, dq or None, dlocal_k or None, dlocal_v or None,
                                         dbank_k or None, dbank_v or None, stream or None)
    if check:
        _check(st, "msa_attend_backward_saved")
    return st


def msa_set_kv_cache(bank, nbytes: int, check=True) -> int:
    st = lib().msa_set_kv_cache(bank, int(nbytes))
    if check:
        _check(st, "msa_set_kv_cache")
    return st


def msa_kv_cache_stats(bank) -> dict:
    vals = [ctypes.c_int64() for _ in range(3)]
    _check(lib().msa_kv_cache_stats(bank, *[ctypes.byref(v) for v in vals]), "msa_kv_cache_stats")
    return {"slabs": vals[0].value, "hits": vals[1].value, "bytes_copied": vals[2].value}


def msa_set_host_fetch(bank, mode: int, check=True) -> int:
    """MSA_FETCH_SM_GATHER (default where the host K/V is mapped) or MSA_FETCH_COPY_ENGINE."""
    st = lib().msa_set_host_fetch(bank, int(mode))
    if check:
        _check(st, "msa_set_host_fetch")
    return st


def msa_get_host_fetch(bank) -> int:
    v = ctypes.c_int()
    _check(lib().msa_get_host_fetch(bank, ctypes.byref(v)), "msa_get_host_fetch")
    return v.value


def msa_set_router_precision(bank, precision: int) -> None:
    """MSA_KR_F32 (default: K_r hi + lo, ~16 significant bits) or MSA_KR_BF16 (the bf16 high part only)."""
    _check(lib().msa_set_router_precision(bank, int(precision)), "msa_set_router_precision")


def msa_check_wait_timeout(bank, stream=0) -> None:
    _check(lib().msa_check_wait_timeout(bank, stream or None), "msa_check_wait_timeout")


def msa_get_device_error(bank, stream=0) -> int:
    return lib().msa_get_device_error(bank, stream or None)


def msa_bank_set_shard(bank, doc_base: int, n_docs_total: int, max_doc_len_total: int, check=True) -> int:
    """Marks the bank as documents [doc_base, doc_base + n_docs) of an n_docs_total-document bank."""
    st = lib().msa_bank_set_shard(bank, int(doc_base), int(n_docs_total), int(max_doc_len_total))
    if check:
        _check(st, "msa_bank_set_shard")
    return st


def msa_attend_partial(bank, query: msa_query, top_k: int, topk_idx: int, with_local: int, out: int, lse: int,
                       stream=0, check=True) -> int:
    st = lib().msa_attend_partial(bank, ctypes.byref(query), top_k, topk_idx or None, int(with_local), out or None,
                                  lse or None, stream or None)
    if check:
        _check(st, "msa_attend_partial")
    return st


def msa_merge_topk(n_parts: int, rows: int, top_k: int, cand_scores: int, cand_idx: int, topk_idx: int,
                   topk_scores: int, stream=0, check=True) -> int:
    st = lib().msa_merge_topk(int(n_parts), int(rows), int(top_k), cand_scores or None, cand_idx or None,
                              topk_idx or None, topk_scores or None, stream or None)
    if check:
        _check(st, "msa_merge_topk")
    return st


def msa_merge_partials(n_parts: int, rows: int, head_dim: int, part_out: int, part_lse: int, out: int, lse: int,
                       stream=0, check=True) -> int:
    st = lib().msa_merge_partials(int(n_parts), int(rows), int(head_dim), part_out or None, part_lse or None,
                                  out or None, lse or None, stream or None)
    if check:
        _check(st, "msa_merge_partials")
    return st


def msa_interleave_route(bank, query: msa_query, top_k: int, q_r_in: int, context_idx: int, n_ctx: int,
                         ctx_out: int, topk_scores: int, q_r_out: int, stream=0, check=True) -> int:
    """One Memory Interleave hop: route over the documents outside the context, expand it, next query."""
    st = lib().msa_interleave_route(bank, ctypes.byref(query), int(top_k), q_r_in or None, context_idx or None,
                                    int(n_ctx), ctx_out or None, topk_scores or None, q_r_out or None, stream or None)
    if check:
        _check(st, "msa_interleave_route")
    return st


def msa_selftest_exp2_poly(x: int, y_poly: int, y_lib: int, n: int, stream=0) -> None:
    """Self-test hook: the prefill kernel's polynomial 2^x and CUDA's exp2f over x [n] (device fp32)."""
    _check(lib().msa_selftest_exp2_poly(x or None, y_poly or None, y_lib or None, int(n), stream or None),
           "msa_selftest_exp2_poly")


def msa_selftest_topk(scores: int, rows: int, n: int, k: int, idx: int, top_scores: int = 0, path: int = 0,
                      stream=0, check=True) -> int:
    """Self-test hook: top-k of [rows][n] device fp32 scores by the chosen kernel (0 auto, 1 block, 2 warp)."""
    st = lib().msa_selftest_topk(scores or None, int(rows), int(n), int(k), idx or None, top_scores or None,
                                 int(path), stream or None)
    if check:
        _check(st, "msa_selftest_topk")
    return st
