"""Convenience layer over the C ABI for torch-held buffers (marshalling only).

Bank: creates a bank handle over device (or pinned-host) K/V tensors and runs
msa_build_bank. step(): one routed step through msa_forward. All arithmetic
happens inside libmsa.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (MSA_DTYPE_BF16, MSA_DTYPE_F32, MSA_KV_DEVICE, make_query, msa_attend, msa_bank_create,
               msa_bank_destroy, msa_bank_info, msa_bank_set_shard, msa_build_bank, msa_forward, msa_get_device_error,
               msa_get_host_fetch, msa_kv_cache_stats, msa_reserve, msa_route, msa_set_host_fetch, msa_set_kv_cache,
               msa_set_router_precision, ptr)


class _DeviceArray:
    """A read-only view of library-owned device memory for torch.as_tensor."""

    def __init__(self, p: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (p, False),
                                         "version": 2}


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Bank:
    """A bank over [Hkv, rows, d] K/V tensors, bf16 or fp32 (the bank's element type
    follows K; K gets Parallel RoPE in place on build)."""

    def __init__(self, K: torch.Tensor, V: torch.Tensor, doc_lens, rope_base: float = 10000.0,
                 kv_location: int = MSA_KV_DEVICE, doc_rows=None):
        assert K.dtype in (torch.bfloat16, torch.float32) and V.dtype == K.dtype and K.shape == V.shape
        self.K, self.V = K, V
        self.dtype = K.dtype
        self.n_kv_heads, self.kv_rows, self.head_dim = K.shape
        self.doc_lens = np.asarray(doc_lens, dtype=np.int64)
        _, self.handle = msa_bank_create(len(self.doc_lens), self.n_kv_heads, self.head_dim, self.doc_lens,
                                         ptr(K), ptr(V), rope_base, kv_location, self.kv_rows, doc_rows,
                                         dtype=MSA_DTYPE_F32 if K.dtype == torch.float32 else MSA_DTYPE_BF16)
        self.info = msa_bank_info(self.handle)

    def build(self, R: torch.Tensor, doc_begin: int = 0, doc_end=None, K_slice=None, stream=None,
              rope: bool = True):
        """Pools K_r from R [Hkv, T, d_r] of docs [doc_begin, doc_end); RoPEs K_slice
        (default: the bank's own K rows of those documents) in place unless rope=False."""
        doc_end = len(self.doc_lens) if doc_end is None else doc_end
        off = np.concatenate([[0], np.cumsum(self.doc_lens)])
        tok0 = int(off[doc_begin])
        if not rope:
            k_ptr, k_stride = 0, 0
        elif K_slice is None:
            K_slice = self.K
            k_ptr = self.K.data_ptr() + tok0 * self.head_dim * self.K.element_size()
            k_stride = self.kv_rows
        else:
            k_ptr = ptr(K_slice, self.dtype)
            k_stride = K_slice.shape[1]
        if R is not None:
            assert R.is_contiguous() and R.dtype == self.dtype
        msa_build_bank(self.handle, doc_begin, doc_end, 0 if R is None else R.data_ptr(),
                       0 if R is None else R.shape[1], k_ptr, k_stride, _stream(stream))

    def k_r(self) -> torch.Tensor:
        """A copy of K_r [Hkv, n_chunks, d_r] fp32 (device)."""
        shape = (self.n_kv_heads, self.info["n_chunks"], self.head_dim)
        return torch.as_tensor(_DeviceArray(self.info["k_r"], shape, "<f4"), device="cuda").clone()

    def k_r_inv_norm(self) -> torch.Tensor:
        shape = (self.n_kv_heads, self.info["n_chunks"])
        return torch.as_tensor(_DeviceArray(self.info["k_r_inv_norm"], shape, "<f4"), device="cuda").clone()

    def query(self, Q, Qr, LK, LV, route_block: int):
        B, Hq, Tq, _ = Q.shape
        return make_query(B, Hq, Tq, LK.shape[2], route_block, ptr(Q, self.dtype),
                          ptr(Qr, self.dtype), ptr(LK, self.dtype), ptr(LV, self.dtype))

    def reserve(self, query, top_k):
        msa_reserve(self.handle, query, top_k)

    def route(self, query, top_k, want_scores=True, stream=None):
        B, Hq, Tq, Lc, Bq = query.batch, query.n_q_heads, query.q_tokens, query.local_len, query.route_block
        nblk = Tq // Bq
        dev = torch.device("cuda")
        idx = torch.empty((B, nblk, self.n_kv_heads, top_k), dtype=torch.int32, device=dev)
        tsc = torch.empty((B, nblk, self.n_kv_heads, top_k), dtype=torch.float32, device=dev)
        scores = (torch.empty((B, nblk, self.n_kv_heads, len(self.doc_lens)), dtype=torch.float32, device=dev)
                  if want_scores else None)
        msa_route(self.handle, query, top_k, ptr(scores), ptr(idx), ptr(tsc), _stream(stream))
        return idx, tsc, scores

    def attend(self, query, top_k, idx, out=None, stream=None):
        if out is None:
            out = torch.empty((query.batch, query.n_q_heads, query.q_tokens, self.head_dim),
                              dtype=torch.float32, device="cuda")
        msa_attend(self.handle, query, top_k, ptr(idx, torch.int32), ptr(out), _stream(stream))
        return out

    def forward(self, query, top_k, idx=None, out=None, stream=None):
        nblk = query.q_tokens // query.route_block
        if idx is None:
            idx = torch.empty((query.batch, nblk, self.n_kv_heads, top_k), dtype=torch.int32, device="cuda")
        if out is None:
            out = torch.empty((query.batch, query.n_q_heads, query.q_tokens, self.head_dim),
                              dtype=torch.float32, device="cuda")
        msa_forward(self.handle, query, top_k, ptr(idx, torch.int32), ptr(out), _stream(stream))
        return idx, out

    def set_shard(self, doc_base: int, n_docs_total: int, max_doc_len_total: int):
        """This bank holds documents [doc_base, doc_base + n_docs) of a larger bank (Memory Parallel)."""
        msa_bank_set_shard(self.handle, doc_base, n_docs_total, max_doc_len_total)

    def set_kv_cache(self, nbytes: int):
        """Device-resident slab cache of a pinned-host bank (0 turns it off)."""
        msa_set_kv_cache(self.handle, nbytes)

    def set_router_precision(self, precision: int):
        """MSA_KR_F32 (default) or MSA_KR_BF16: the precision of the routing keys the router reads."""
        msa_set_router_precision(self.handle, precision)

    def set_host_fetch(self, mode: int):
        """MSA_FETCH_SM_GATHER or MSA_FETCH_COPY_ENGINE: how a pinned-host bank moves its slabs."""
        msa_set_host_fetch(self.handle, mode)

    def host_fetch(self) -> int:
        return msa_get_host_fetch(self.handle)

    def cache_stats(self) -> dict:
        """Distinct slabs, cache hits and PCIe bytes of the last host-tier step."""
        return msa_kv_cache_stats(self.handle)

    def device_error(self, stream=None) -> int:
        return msa_get_device_error(self.handle, _stream(stream))

    def close(self):
        if self.handle:
            msa_bank_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
