"""Memory Parallel: one routed step over a bank whose documents are split into
contiguous shards, one shard per device ("MSA架构：突破大模型记忆瓶颈的稀疏注意力技术",
§2.1 item 3: distributed memory retrieval across GPUs through an AllGather;
"MSA (Memory Sparse Attention)", robocikowo.com, Równoległość: the router's scoring
spread over devices, the top-k selection and the K/V fetch following in sequence).

A step:
  1. every shard routes over its own documents (msa_route on a bank marked with
     msa_bank_set_shard): its top_k candidates, scores and global indices;
  2. the candidates are all-gathered (k x 8 bytes per routing row and KV head);
  3. every shard merges them into the global top_k (msa_merge_topk), so all shards
     hold the selection one bank with every document would make;
  4. every shard attends over the selected documents it holds, the owner of the
     sequences also over their local context (msa_attend_partial);
  5. the partials (out, log-sum-exp) are all-gathered and the owner merges them
     (msa_merge_partials).

This module is argument marshalling and collectives only: routing, both merges
and attention run in libmsa. The collectives are torch.distributed all-gathers
(NCCL between GPUs; gloo works for the host-side exchange on CPU tensors); no
device reads another device's memory. `ShardedStep` runs the same five steps for
several shard banks that share one GPU, with tensor stacking in place of the
all-gathers.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import msa_attend_partial, msa_merge_partials, msa_merge_topk, msa_route


def shard_ranges(n_docs: int, n_shards: int) -> List[Tuple[int, int]]:
    """[lo, hi) of n_shards contiguous document ranges whose sizes differ by at most
    one; the first n_docs % n_shards ranges hold one document more."""
    if not 1 <= n_shards <= n_docs:
        raise ValueError("need 1 <= n_shards <= n_docs")
    base, extra = divmod(n_docs, n_shards)
    bounds = [0]
    for s in range(n_shards):
        bounds.append(bounds[-1] + base + (s < extra))
    return list(zip(bounds[:-1], bounds[1:]))


def all_gather_stacked(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's tensor, in rank order (torch.distributed)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def exchange_candidates(scores: torch.Tensor, idx: torch.Tensor, group=None):
    """All-gather of one shard's routing candidates: ([W, rows, k] scores, [W, rows, k] indices)."""
    return all_gather_stacked(scores, group), all_gather_stacked(idx, group)


def exchange_partials(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather of one shard's partial attention: ([W, ...out], [W, ...lse])."""
    return all_gather_stacked(out, group), all_gather_stacked(lse, group)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _route(bank, qry, top_k: int, sh: int):
    nblk = qry.q_tokens // qry.route_block
    shape = (qry.batch, nblk, bank.n_kv_heads, top_k)
    idx = torch.empty(shape, dtype=torch.int32, device="cuda")
    sc = torch.empty(shape, dtype=torch.float32, device="cuda")
    msa_route(bank.handle, qry, top_k, 0, idx.data_ptr(), sc.data_ptr(), sh)
    return sc, idx


def _merge_topk(cand_sc: torch.Tensor, cand_ix: torch.Tensor, top_k: int, sh: int) -> torch.Tensor:
    parts = cand_sc.shape[0]
    rows = cand_sc[0].numel() // top_k
    idx = torch.empty(cand_sc.shape[1:], dtype=torch.int32, device=cand_sc.device)
    msa_merge_topk(parts, rows, top_k, cand_sc.data_ptr(), cand_ix.data_ptr(), idx.data_ptr(), 0, sh)
    return idx


def _partial(bank, qry, top_k: int, idx: torch.Tensor, with_local: bool, sh: int):
    out = torch.empty((qry.batch, qry.n_q_heads, qry.q_tokens, bank.head_dim), dtype=torch.float32, device="cuda")
    lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
    msa_attend_partial(bank.handle, qry, top_k, idx.data_ptr(), int(with_local), out.data_ptr(), lse.data_ptr(), sh)
    return out, lse


def _merge_partials(parts_out: torch.Tensor, parts_lse: torch.Tensor, sh: int) -> torch.Tensor:
    n, d = parts_out.shape[0], parts_out.shape[-1]
    out = torch.empty(parts_out.shape[1:], dtype=torch.float32, device=parts_out.device)
    msa_merge_partials(n, parts_lse[0].numel(), d, parts_out.data_ptr(), parts_lse.data_ptr(), out.data_ptr(), 0, sh)
    return out


class MemoryParallelStep:
    """One rank's part of a Memory Parallel step (one process per GPU).

    `bank` is this rank's shard (a runner.Bank marked with msa_bank_set_shard); every
    rank passes its own msa_query over the same sequences (the routing queries are
    needed everywhere; the queries and the local K/V only matter on the owner).
    Returns (the global selection, the output on the owner / None elsewhere)."""

    def __init__(self, bank, owner: int = 0, group=None):
        import torch.distributed as dist
        self.bank, self.owner, self.group = bank, owner, group
        self.rank = dist.get_rank(group)

    def __call__(self, qry, top_k: int, stream=None):
        sh = _stream(stream)
        sc, ix = _route(self.bank, qry, top_k, sh)
        all_sc, all_ix = exchange_candidates(sc, ix, self.group)
        idx = _merge_topk(all_sc, all_ix, top_k, sh)
        out, lse = _partial(self.bank, qry, top_k, idx, self.rank == self.owner, sh)
        all_out, all_lse = exchange_partials(out, lse, self.group)
        return idx, (_merge_partials(all_out, all_lse, sh) if self.rank == self.owner else None)


class ShardedStep:
    """The Memory Parallel step for several shard banks on one GPU: the all-gathers
    become stacks of the shards' device tensors; the routing, merges and attention
    are the same library calls as MemoryParallelStep's. `queries[s]` is shard s's
    msa_query (the same sequences; shard `owner` attends the local context)."""

    def __init__(self, banks: Sequence, owner: int = 0):
        self.banks, self.owner = list(banks), owner

    def __call__(self, queries: Sequence, top_k: int, stream=None, parts: bool = False):
        sh = _stream(stream)
        cands = [_route(b, q, top_k, sh) for b, q in zip(self.banks, queries)]
        idx = _merge_topk(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]), top_k, sh)
        partials = [_partial(b, q, top_k, idx, s == self.owner, sh)
                    for s, (b, q) in enumerate(zip(self.banks, queries))]
        out = _merge_partials(torch.stack([p[0] for p in partials]), torch.stack([p[1] for p in partials]), sh)
        if parts:
            return idx, out, cands, partials
        return idx, out


def shard_bank_tensors(K: torch.Tensor, V: torch.Tensor, R: Optional[torch.Tensor], doc_lens,
                       ranges: Sequence[Tuple[int, int]]):
    """Per-shard contiguous copies [Hkv, rows of the shard's documents, d] of a bank's
    K, V and routing keys R (documents concatenated in order)."""
    off = np.concatenate([[0], np.cumsum(np.asarray(doc_lens, dtype=np.int64))])
    out = []
    for lo, hi in ranges:
        a, b = int(off[lo]), int(off[hi])
        out.append((K[:, a:b].contiguous(), V[:, a:b].contiguous(), None if R is None else R[:, a:b].contiguous()))
    return out
