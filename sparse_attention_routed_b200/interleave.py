"""Memory Interleave: routing in hops that expand the context ("MSA (Memory Sparse
Attention)", robocikowo.com, Komponenty: document identifiers and context expansion
alternate; "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §3.2: retrieval in rounds).

Each hop is one msa_interleave_route call (route over the documents not yet in the
context, append the hop's top_k, form the next routing query) and one msa_attend
over the whole expanded context. Argument marshalling only: the routing, the
context update, the query update and the attention run in libmsa; torch holds the
buffers.
"""
from __future__ import annotations

from typing import List, Tuple

import torch

from . import msa_attend, msa_interleave_route


def run_hops(bank, qry, top_k: int, hops: int, stream=None) -> List[Tuple[torch.Tensor, torch.Tensor]]:
    """Runs `hops` hops for the step described by `qry` on `bank` (a runner.Bank).
    Returns, per hop, (the expanded context [B, nblk, Hkv, (t+1) * top_k] int32,
    the attention output over it [B, Hq, Tq, d] fp32)."""
    sh = (stream if stream is not None else torch.cuda.current_stream()).cuda_stream
    nblk = qry.q_tokens // qry.route_block
    B, Hkv, d = qry.batch, bank.n_kv_heads, bank.head_dim
    q_in = None
    ctx = None
    res = []
    for t in range(hops):
        n_ctx = t * top_k
        ctx_out = torch.empty((B, nblk, Hkv, n_ctx + top_k), dtype=torch.int32, device="cuda")
        q_out = torch.empty((B, Hkv, nblk, d), dtype=torch.float32, device="cuda") if t + 1 < hops else None
        msa_interleave_route(bank.handle, qry, top_k, 0 if q_in is None else q_in.data_ptr(),
                             0 if ctx is None else ctx.data_ptr(), n_ctx, ctx_out.data_ptr(), 0,
                             0 if q_out is None else q_out.data_ptr(), sh)
        out = torch.empty((B, qry.n_q_heads, qry.q_tokens, d), dtype=torch.float32, device="cuda")
        msa_attend(bank.handle, qry, n_ctx + top_k, ctx_out.data_ptr(), out.data_ptr(), sh)
        res.append((ctx_out, out))
        ctx, q_in = ctx_out, q_out
    return res
