"""CPU oracle of the routed sparse-attention step of Memory Sparse Attention (MSA).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code,
table or helper with the CUDA library, and the library never calls it.

Everything is plain numpy in fp64, one document / one chunk / one query row at
a time, in the order the method states its steps:

1. chunk-mean pooling of each document's per-token routing keys into the
   compressed routing keys K_r (256-token chunks)
   -- "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 2 and §3.1
      (the ``chunk_mean_pooling`` example: a mean over each 256-token chunk);
   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty: the
      Router's K_r is a compressed document representation; Pułapki
      implementacyjne: build the bank offline with chunked mean pooling.
2. Parallel (document-wise) RoPE on the bank keys: positions restart at 0 at
   every document's first token
   -- "MSA架构…", §2.2; robocikowo.com, Komponenty (Document-wise RoPE,
      Parallel RoPE) and Pułapki implementacyjne (RoPE consistency).
3. the routing query q_r of a query block = mean of its tokens' routing queries.
4. router: cosine similarity between q_r and every chunk of K_r; a document's
   score is the max over its chunks
   -- "MSA架构…", §2.1 item 1 (cosine top-k router); robocikowo.com,
      Komponenty (Router / Routing Projector).
5. top-k documents per (query block, KV head), larger score first, equal
   scores to the lower document index
   -- robocikowo.com, Hiperparametry (Top-k documents), Paradygmat wykonania.
6. one softmax attention over the selected documents' K/V (all visible) plus
   the causal local context, whose queries and keys carry Global RoPE at
   positions k_off + u with k_off = top_k * max document length
   -- robocikowo.com, Komponenty (Memory Sparse Attention Layer: append the
      selected documents' K/V to the local context; Global RoPE), Pułapki
      implementacyjne (Global RoPE with a k-offset for the active context),
      Paradygmat wykonania (only the k selected documents take part).

Readings where the pages are silent:
the document score is the max over its chunks; a ragged last chunk is the mean
over its actual tokens; q_r is the unnormalised block mean; a zero-norm cosine
is 0; RoPE is rotate-half with theta_i = base^(-2i/d); the softmax scale is
1/sqrt(d); query head hq reads KV head hq // (Hq/Hkv); the Tq queries are the
last Tq local tokens and local key u is visible to local query i iff u <= i.

Parity pins: every function here is pinned -- tests/test_oracle_pins.py (the
step), tests/test_oracle_backward.py (the backward), tests/test_oracle_router_bf16.py
(the bf16-key router variant), tests/test_oracle_lse.py (the row log-sum-exp),
tests/test_oracle_memory_parallel.py (the document-sharded step) and
tests/test_oracle_interleave.py (multi-hop Memory Interleave) -- against closed
forms, invariants, library special cases or brute force.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

CHUNK = 256


# --------------------------------------------------------------------------
# 1. document layout and chunk-mean pooling
# --------------------------------------------------------------------------

def doc_offsets(doc_lens: Sequence[int]) -> np.ndarray:
    """Token offset of every document in the concatenated bank, length n+1."""
    off = np.zeros(len(doc_lens) + 1, dtype=np.int64)
    for j, L in enumerate(doc_lens):
        if L < 1:
            raise ValueError("every document holds at least one token")
        off[j + 1] = off[j] + int(L)
    return off


def chunk_spans(doc_len: int, chunk: int = CHUNK) -> List[Tuple[int, int]]:
    """[start, end) token spans of one document's chunks, relative to the document."""
    return [(s, min(s + chunk, doc_len)) for s in range(0, doc_len, chunk)]


def chunk_mean_pool(R_doc: np.ndarray, chunk: int = CHUNK) -> np.ndarray:
    """K_r rows of one document: the arithmetic mean of each chunk's actual tokens.

    R_doc: [L, d_r] per-token routing keys of one document and one KV head.
    Returns [ceil(L/chunk), d_r] in fp64.
    """
    R_doc = np.asarray(R_doc, dtype=np.float64)
    rows = []
    for s, e in chunk_spans(R_doc.shape[0], chunk):
        total = np.zeros(R_doc.shape[1], dtype=np.float64)
        for t in range(s, e):
            total += R_doc[t]
        rows.append(total / (e - s))
    return np.stack(rows)


def build_routing_keys(R_head: np.ndarray, doc_lens: Sequence[int],
                       chunk: int = CHUNK) -> Tuple[np.ndarray, np.ndarray]:
    """K_r of one KV head over the whole bank.

    R_head: [Ntok, d_r] routing keys of one KV head, documents concatenated.
    Returns (K_r [Nch, d_r], chunk_doc [Nch]) where chunk_doc[c] is the
    document that owns chunk c.
    """
    off = doc_offsets(doc_lens)
    kr, owner = [], []
    for j, L in enumerate(doc_lens):
        rows = chunk_mean_pool(R_head[off[j]:off[j + 1]], chunk)
        kr.append(rows)
        owner.extend([j] * rows.shape[0])
    return np.concatenate(kr, axis=0), np.asarray(owner, dtype=np.int64)


# --------------------------------------------------------------------------
# 2. RoPE (rotate-half), Parallel and Global placement
# --------------------------------------------------------------------------

def rope_inv_freq(d: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d), i < d/2, in fp64."""
    i = np.arange(d // 2, dtype=np.float64)
    return base ** (-2.0 * i / d)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE: pair (x_i, x_{i+d/2}) is turned by pos * theta_i.

    x: [..., d]; pos: scalar or array broadcastable to x.shape[:-1].
    x'_i = x_i cos - x_{i+d/2} sin;  x'_{i+d/2} = x_{i+d/2} cos + x_i sin.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def parallel_rope_positions(doc_lens: Sequence[int]) -> np.ndarray:
    """Position of every bank token: its index inside its own document."""
    return np.concatenate([np.arange(int(L), dtype=np.int64) for L in doc_lens])


def parallel_rope_bank(K_head: np.ndarray, doc_lens: Sequence[int], base: float) -> np.ndarray:
    """Bank keys of one KV head with document-wise (Parallel) RoPE applied."""
    return rope(K_head, parallel_rope_positions(doc_lens), base)


def k_offset(top_k: int, doc_lens: Sequence[int]) -> int:
    """Global-RoPE offset of the active context: top_k * (longest document)."""
    return int(top_k) * int(max(int(L) for L in doc_lens))


# --------------------------------------------------------------------------
# 3-5. routing
# --------------------------------------------------------------------------

def block_mean_query(Qr_tokens: np.ndarray, route_block: int) -> np.ndarray:
    """q_r of each routing block: mean of its tokens' routing queries.

    Qr_tokens: [Tq, d_r] for one (sequence, KV head). Returns [Tq/route_block, d_r].
    """
    Qr_tokens = np.asarray(Qr_tokens, dtype=np.float64)
    Tq = Qr_tokens.shape[0]
    if Tq % route_block:
        raise ValueError("query tokens must split into whole routing blocks")
    out = []
    for s in range(0, Tq, route_block):
        total = np.zeros(Qr_tokens.shape[1], dtype=np.float64)
        for t in range(s, s + route_block):
            total += Qr_tokens[t]
        out.append(total / route_block)
    return np.stack(out)


def cosine(q: np.ndarray, k: np.ndarray) -> float:
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    den = math.sqrt(float(q @ q)) * math.sqrt(float(k @ k))
    return float(q @ k) / max(den, 1e-30)


def route_doc_scores(q_r: np.ndarray, K_r: np.ndarray, chunk_doc: np.ndarray,
                     n_docs: int) -> np.ndarray:
    """Document scores of one routing query: max over each document's chunk cosines."""
    scores = np.full(n_docs, -np.inf, dtype=np.float64)
    for c in range(K_r.shape[0]):
        s = cosine(q_r, K_r[c])
        j = int(chunk_doc[c])
        if s > scores[j]:
            scores[j] = s
    return scores


def chunk_cosines(q_r: np.ndarray, K_r: np.ndarray) -> np.ndarray:
    """All chunk cosines of one routing query at once (same definition, vectorised)."""
    q = np.asarray(q_r, dtype=np.float64)
    K = np.asarray(K_r, dtype=np.float64)
    den = np.sqrt(q @ q) * np.sqrt(np.einsum("cd,cd->c", K, K))
    return (K @ q) / np.maximum(den, 1e-30)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> the nearest bf16 value (8 significant bits, ties to even), as fp64.
    x = m 2^e with 1/2 <= |m| < 1; m 2^8 rounded to an integer (half to even)."""
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.rint(m * 256.0), e - 8)


def chunk_cosines_bf16_keys(q_r: np.ndarray, K_r: np.ndarray) -> np.ndarray:
    """Chunk cosines with the normalised routing keys stored in bf16 (the reduced-
    precision router variant): q^ . bf16(k^), q^ = q_r / |q_r| and k^ = K_r / |K_r|
    exact. Differs from the exact cosine by at most 2^-8 sum_i |q^_i k^_i| <= 2^-8."""
    q = np.asarray(q_r, dtype=np.float64)
    K = np.asarray(K_r, dtype=np.float64)
    qh = q / max(math.sqrt(float(q @ q)), 1e-30)
    kh = K / np.maximum(np.sqrt(np.einsum("cd,cd->c", K, K)), 1e-30)[:, None]
    return round_bf16(kh) @ qh


def doc_max(chunk_scores: np.ndarray, chunk_doc: np.ndarray, n_docs: int) -> np.ndarray:
    out = np.full(n_docs, -np.inf, dtype=np.float64)
    np.maximum.at(out, chunk_doc, chunk_scores)
    return out


def select_top_k(doc_scores: np.ndarray, top_k: int) -> np.ndarray:
    """Indices of the top_k documents, ordered by (score desc, index asc)."""
    n = len(doc_scores)
    if not 1 <= top_k <= n:
        raise ValueError("1 <= top_k <= n_docs")
    order = sorted(range(n), key=lambda j: (-float(doc_scores[j]), j))
    return np.asarray(order[:top_k], dtype=np.int64)


# --------------------------------------------------------------------------
# 6. routed attention
# --------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray) -> np.ndarray:
    """softmax(q . keys^T / sqrt(d)) . values for one query row, fp64, max-subtracted."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    logits = (np.asarray(keys, dtype=np.float64) @ q) / math.sqrt(d)
    m = logits.max()
    w = np.exp(logits - m)
    return (w @ np.asarray(values, dtype=np.float64)) / w.sum()


def routed_attention_row(q: np.ndarray, q_index: int, k_off: int, base: float,
                         mem_k_rot: np.ndarray, mem_v: np.ndarray,
                         local_k: np.ndarray, local_v: np.ndarray) -> np.ndarray:
    """Output of one query row.

    q:        [d] un-rotated query of the local token at index q_index.
    mem_k_rot:[M, d] keys of the selected documents with Parallel RoPE applied.
    mem_v:    [M, d] their values.
    local_k/v:[Lc, d] un-rotated local keys / values; keys 0..q_index are visible.
    """
    q_rot = rope(q, k_off + q_index, base)
    vis = q_index + 1
    loc_k_rot = rope(local_k[:vis], k_off + np.arange(vis), base)
    keys = np.concatenate([np.asarray(mem_k_rot, dtype=np.float64), loc_k_rot], axis=0)
    values = np.concatenate([np.asarray(mem_v, dtype=np.float64),
                             np.asarray(local_v[:vis], dtype=np.float64)], axis=0)
    return softmax_attention(q_rot, keys, values)


def routed_attention_row_lse(q: np.ndarray, q_index: int, k_off: int, base: float,
                             mem_k_rot: np.ndarray, local_k: np.ndarray) -> float:
    """log sum_j exp(s_j) (natural log) over one query row's key set, with
    s_j = q_rot . k_j / sqrt(d) -- the normaliser of routed_attention_row's softmax
    (out = sum_j exp(s_j - lse) v_j). Same key set and RoPE positions; evaluated as
    m + log sum_j exp(s_j - m), m = max_j s_j."""
    q_rot = rope(q, k_off + q_index, base)
    d = q_rot.shape[-1]
    vis = q_index + 1
    loc_k_rot = rope(local_k[:vis], k_off + np.arange(vis), base)
    keys = np.concatenate([np.asarray(mem_k_rot, dtype=np.float64), loc_k_rot], axis=0)
    s = keys @ q_rot / math.sqrt(d)
    m = s.max()
    return float(m + math.log(np.exp(s - m).sum()))


# --------------------------------------------------------------------------
# the whole step on explicit (small) tensors
# --------------------------------------------------------------------------

def forward(inputs: Dict[str, np.ndarray], doc_lens: Sequence[int], top_k: int,
            route_block: int, base: float = 10000.0, chunk: int = CHUNK,
            selection=None, router_keys: str = "f32") -> Dict[str, np.ndarray]:
    """The routed sparse-attention step on fully materialised inputs.

    inputs (all real-valued arrays, converted to fp64):
      K, V   [Hkv, Ntok, d]  bank keys (un-rotated) and values
      R      [Hkv, Ntok, d_r] per-token routing keys
      Q      [B, Hq, Tq, d]  un-rotated queries (the last Tq local tokens)
      Qr     [B, Hkv, Tq, d_r] per-token routing queries
      LK, LV [B, Hkv, Lc, d] un-rotated local keys / values
    selection: optional [B, nblk, Hkv, k] document indices to attend over
      instead of the oracle's own top-k (used when several sets are correct).
    router_keys: "f32" (the exact cosine) or "bf16" (the reduced-precision router
      variant: normalised routing keys rounded to bf16, chunk_cosines_bf16_keys).

    Returns K_r [Hkv, Nch, d_r], K_rot [Hkv, Ntok, d], q_r [B, nblk, Hkv, d_r],
    doc_scores [B, nblk, Hkv, n], topk [B, nblk, Hkv, k], out [B, Hq, Tq, d].
    """
    K = np.asarray(inputs["K"], dtype=np.float64)
    V = np.asarray(inputs["V"], dtype=np.float64)
    R = np.asarray(inputs["R"], dtype=np.float64)
    Q = np.asarray(inputs["Q"], dtype=np.float64)
    Qr = np.asarray(inputs["Qr"], dtype=np.float64)
    LK = np.asarray(inputs["LK"], dtype=np.float64)
    LV = np.asarray(inputs["LV"], dtype=np.float64)
    Hkv, Ntok, d = K.shape
    B, Hq, Tq, _ = Q.shape
    Lc = LK.shape[2]
    n = len(doc_lens)
    G = Hq // Hkv
    nblk = Tq // route_block
    off = doc_offsets(doc_lens)
    k_off = k_offset(top_k, doc_lens)

    K_r, chunk_doc = [], None
    K_rot = np.empty_like(K)
    for h in range(Hkv):
        kr, chunk_doc = build_routing_keys(R[h], doc_lens, chunk)
        K_r.append(kr)
        K_rot[h] = parallel_rope_bank(K[h], doc_lens, base)
    K_r = np.stack(K_r)

    q_r = np.empty((B, nblk, Hkv, R.shape[2]))
    scores = np.empty((B, nblk, Hkv, n))
    topk = np.empty((B, nblk, Hkv, top_k), dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            qb = block_mean_query(Qr[b, h], route_block)
            for blk in range(nblk):
                q_r[b, blk, h] = qb[blk]
                if router_keys == "bf16":
                    scores[b, blk, h] = doc_max(chunk_cosines_bf16_keys(qb[blk], K_r[h]), chunk_doc, n)
                else:
                    scores[b, blk, h] = route_doc_scores(qb[blk], K_r[h], chunk_doc, n)
                topk[b, blk, h] = select_top_k(scores[b, blk, h], top_k)
    sel = topk if selection is None else np.asarray(selection, dtype=np.int64)

    out = np.empty((B, Hq, Tq, d))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for t in range(Tq):
                blk = t // route_block
                docs = sel[b, blk, h]
                mk = np.concatenate([K_rot[h, off[j]:off[j + 1]] for j in docs], axis=0)
                mv = np.concatenate([V[h, off[j]:off[j + 1]] for j in docs], axis=0)
                i = Lc - Tq + t
                out[b, hq, t] = routed_attention_row(Q[b, hq, t], i, k_off, base, mk, mv,
                                                     LK[b, h], LV[b, h])
    return {"K_r": K_r, "K_rot": K_rot, "q_r": q_r, "doc_scores": scores, "topk": topk,
            "out": out, "k_off": k_off}


# --------------------------------------------------------------------------
# backward of the routed attention (the selection is fixed: top-k routing is
# not differentiated), for training the layer end to end
#   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty: the memory
#      sparse attention layer is trained end to end on top of a fixed router
#      selection per step.
# --------------------------------------------------------------------------

def rope_adjoint(g: np.ndarray, pos, base: float) -> np.ndarray:
    """Adjoint (transpose) of rope at the same positions: the inverse rotation,
    i.e. a turn by -pos * theta_i (each pair's rotation matrix is orthogonal)."""
    return rope(g, -np.asarray(pos, dtype=np.float64), base)


def routed_attention_row_backward(q: np.ndarray, q_index: int, k_off: int, base: float,
                                  mem_k_rot: np.ndarray, mem_v: np.ndarray,
                                  local_k: np.ndarray, local_v: np.ndarray, d_out: np.ndarray):
    """Gradients of sum(d_out * o) for one query row o = routed_attention_row(...).

    With s_j = q_rot . k_j / sqrt(d), p = softmax(s), o = sum_j p_j v_j:
      dv_j = p_j d_out;  dp_j = d_out . v_j;  ds_j = p_j (dp_j - d_out . o);
      dq_rot = sum_j ds_j k_j / sqrt(d);  dk_j = ds_j q_rot / sqrt(d);
    rotated quantities go back through the RoPE adjoint.
    Returns dq (un-rotated), d_mem_k_rot [M, d] (with respect to the rotated bank
    keys), d_mem_v [M, d], d_local_k [vis, d] (un-rotated), d_local_v [vis, d].
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    M = len(mem_k_rot)
    q_rot = rope(q, k_off + q_index, base)
    vis = q_index + 1
    loc_pos = k_off + np.arange(vis)
    loc_k_rot = rope(local_k[:vis], loc_pos, base)
    keys = np.concatenate([np.asarray(mem_k_rot, dtype=np.float64), loc_k_rot], axis=0)
    values = np.concatenate([np.asarray(mem_v, dtype=np.float64),
                             np.asarray(local_v[:vis], dtype=np.float64)], axis=0)
    s = keys @ q_rot / math.sqrt(d)
    w = np.exp(s - s.max())
    p = w / w.sum()
    o = p @ values
    d_out = np.asarray(d_out, dtype=np.float64)
    dp = values @ d_out
    ds = p * (dp - d_out @ o)
    dq_rot = ds @ keys / math.sqrt(d)
    dkeys = np.outer(ds, q_rot) / math.sqrt(d)
    dvalues = np.outer(p, d_out)
    dq = rope_adjoint(dq_rot, k_off + q_index, base)
    d_local_k = rope_adjoint(dkeys[M:], loc_pos, base)
    return dq, dkeys[:M], dvalues[:M], d_local_k, dvalues[M:]


def backward(inputs: Dict[str, np.ndarray], doc_lens: Sequence[int], top_k: int, route_block: int,
             d_out: np.ndarray, base: float = 10000.0, chunk: int = CHUNK, selection=None) -> Dict[str, np.ndarray]:
    """Gradients of L = sum(d_out * out) with respect to Q, the bank keys K and
    values V (K before Parallel RoPE, as msa_build_bank takes them), and the
    local keys LK (before Global RoPE) and values LV, with the step's selection
    held fixed (the oracle's own top-k, or `selection`).

    Returns dQ [B, Hq, Tq, d], dK / dV [Hkv, Ntok, d], dLK / dLV [B, Hkv, Lc, d]
    and the selection used."""
    fwd = forward(inputs, doc_lens, top_k, route_block, base, chunk, selection)
    sel = fwd["topk"] if selection is None else np.asarray(selection, dtype=np.int64)
    K_rot = fwd["K_rot"]
    k_off = fwd["k_off"]
    V = np.asarray(inputs["V"], dtype=np.float64)
    Q = np.asarray(inputs["Q"], dtype=np.float64)
    LK = np.asarray(inputs["LK"], dtype=np.float64)
    LV = np.asarray(inputs["LV"], dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    Hkv, Ntok, d = K_rot.shape
    B, Hq, Tq, _ = Q.shape
    Lc = LK.shape[2]
    G = Hq // Hkv
    off = doc_offsets(doc_lens)

    dQ = np.zeros_like(Q)
    dK_rot = np.zeros((Hkv, Ntok, d))
    dV = np.zeros((Hkv, Ntok, d))
    dLK = np.zeros_like(LK)
    dLV = np.zeros_like(LV)
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for t in range(Tq):
                docs = sel[b, t // route_block, h]
                mk = np.concatenate([K_rot[h, off[j]:off[j + 1]] for j in docs], axis=0)
                mv = np.concatenate([V[h, off[j]:off[j + 1]] for j in docs], axis=0)
                i = Lc - Tq + t
                dq, dmk, dmv, dlk, dlv = routed_attention_row_backward(
                    Q[b, hq, t], i, k_off, base, mk, mv, LK[b, h], LV[b, h], d_out[b, hq, t])
                dQ[b, hq, t] = dq
                row = 0
                for j in docs:
                    L = off[j + 1] - off[j]
                    dK_rot[h, off[j]:off[j + 1]] += dmk[row:row + L]
                    dV[h, off[j]:off[j + 1]] += dmv[row:row + L]
                    row += L
                dLK[b, h, :i + 1] += dlk
                dLV[b, h, :i + 1] += dlv
    # the bank keys were turned by Parallel RoPE (positions restart in every document)
    dK = np.empty_like(dK_rot)
    for h in range(Hkv):
        for j in range(len(doc_lens)):
            L = off[j + 1] - off[j]
            dK[h, off[j]:off[j + 1]] = rope_adjoint(dK_rot[h, off[j]:off[j + 1]], np.arange(L), base)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dLK": dLK, "dLV": dLV, "selection": sel, "out": fwd["out"]}


# --------------------------------------------------------------------------
# Memory Parallel: the bank's documents split into contiguous shards, one per
# device; each shard scores its own documents, the shards' candidates are
# gathered and merged into the one global top-k, each shard attends over the
# selected documents it holds, and the partial attentions are combined
#   -- "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 3 (memory parallel:
#      distributed memory retrieval across GPUs through an AllGather);
#   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Równoległość (the Memory
#      Parallel engine scores the router across devices; the top-k selection and
#      the K/V fetch that follows stay sequential within each decoding step).
# Reading: the gathered items are each shard's own top-k candidates (score,
# global document index); the merge keeps the top_k of their union under the
# single-bank order (score desc, index asc); the partial of a shard is its
# softmax over the keys it holds together with that softmax's log-sum-exp, and
# the local context is attended by one shard (the owner of the sequence).
# --------------------------------------------------------------------------

def shard_ranges(n_docs: int, n_shards: int) -> List[Tuple[int, int]]:
    """[lo, hi) document ranges of n_shards contiguous shards, sizes differing by at
    most one (the first n_docs % n_shards shards hold the extra document)."""
    if not 1 <= n_shards <= n_docs:
        raise ValueError("1 <= n_shards <= n_docs")
    q, r = divmod(n_docs, n_shards)
    out, lo = [], 0
    for s in range(n_shards):
        hi = lo + q + (1 if s < r else 0)
        out.append((lo, hi))
        lo = hi
    return out


def merge_candidates(cand_scores: Sequence[np.ndarray], cand_idx: Sequence[np.ndarray],
                     top_k: int) -> Tuple[np.ndarray, np.ndarray]:
    """The global top_k from the shards' candidate lists: the top_k members of their
    union ordered by (score desc, global index asc). Returns (indices, scores)."""
    pairs = []
    for sc, ix in zip(cand_scores, cand_idx):
        for s, j in zip(np.asarray(sc, dtype=np.float64), np.asarray(ix)):
            pairs.append((-float(s), int(j)))
    if len(pairs) < top_k:
        raise ValueError("fewer candidates than top_k")
    pairs.sort()
    chosen = pairs[:top_k]
    return (np.asarray([j for _, j in chosen], dtype=np.int64),
            np.asarray([-s for s, _ in chosen], dtype=np.float64))


def attention_partial(q_rot: np.ndarray, keys: np.ndarray, values: np.ndarray) -> Tuple[np.ndarray, float]:
    """Attention of one (already rotated) query row over a subset of its keys:
    (softmax over the subset applied to its values, log sum_j exp(s_j) over the
    subset) with s_j = q_rot . k_j / sqrt(d). An empty subset gives (0, -inf)."""
    q = np.asarray(q_rot, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64).reshape(-1, q.shape[-1])
    if keys.shape[0] == 0:
        return np.zeros(q.shape[-1]), -math.inf
    s = keys @ q / math.sqrt(q.shape[-1])
    m = s.max()
    w = np.exp(s - m)
    return (w @ np.asarray(values, dtype=np.float64)) / w.sum(), float(m + math.log(w.sum()))


def merge_partials(outs: Sequence[np.ndarray], lses: Sequence[float]) -> Tuple[np.ndarray, float]:
    """One softmax over the union of disjoint key subsets from their partials:
    L = log sum_s exp(lse_s), out = sum_s exp(lse_s - L) out_s. Parts with
    lse = -inf (no keys) weigh nothing; if every part is empty, (0, -inf)."""
    lses = [float(x) for x in lses]
    finite = [x for x in lses if x != -math.inf]
    if not finite:
        return np.zeros_like(np.asarray(outs[0], dtype=np.float64)), -math.inf
    m = max(finite)
    total = sum(math.exp(x - m) for x in finite)
    L = m + math.log(total)
    out = np.zeros_like(np.asarray(outs[0], dtype=np.float64))
    for o, x in zip(outs, lses):
        if x != -math.inf:
            out = out + math.exp(x - L) * np.asarray(o, dtype=np.float64)
    return out, L


def memory_parallel_forward(inputs: Dict[str, np.ndarray], doc_lens: Sequence[int], top_k: int,
                            route_block: int, n_shards: int, base: float = 10000.0, owner: int = 0,
                            chunk: int = CHUNK) -> Dict[str, np.ndarray]:
    """The routed step of forward() with the documents in n_shards contiguous shards.

    Per (sequence, routing block, KV head): every shard s routes over its own
    documents only (K_r pooled from its routing keys, cosine, max over chunks) and
    keeps its top min(top_k, n_s) (score, global index) candidates; the candidates of
    all shards are merged (merge_candidates). Per query row: every shard attends over
    the merged selection's documents it holds, the owner shard also over the causal
    local context, each giving (out_s, lse_s) (attention_partial); the row's output
    is merge_partials of those. Returns topk [B, nblk, Hkv, k], the candidates
    ([n_shards] lists of [B, nblk, Hkv, k_s] scores / indices), partial outputs and
    log-sum-exps [n_shards, B, Hq, Tq, (d)], and out [B, Hq, Tq, d]."""
    K = np.asarray(inputs["K"], dtype=np.float64)
    V = np.asarray(inputs["V"], dtype=np.float64)
    R = np.asarray(inputs["R"], dtype=np.float64)
    Q = np.asarray(inputs["Q"], dtype=np.float64)
    Qr = np.asarray(inputs["Qr"], dtype=np.float64)
    LK = np.asarray(inputs["LK"], dtype=np.float64)
    LV = np.asarray(inputs["LV"], dtype=np.float64)
    Hkv, _, d = K.shape
    B, Hq, Tq, _ = Q.shape
    Lc = LK.shape[2]
    G = Hq // Hkv
    nblk = Tq // route_block
    n = len(doc_lens)
    off = doc_offsets(doc_lens)
    k_off = k_offset(top_k, doc_lens)          # the whole bank's longest document
    shards = shard_ranges(n, n_shards)

    # each shard's candidates, from its own documents' routing keys
    cand_sc = [np.empty((B, nblk, Hkv, min(top_k, hi - lo))) for lo, hi in shards]
    cand_ix = [np.empty((B, nblk, Hkv, min(top_k, hi - lo)), dtype=np.int64) for lo, hi in shards]
    for s, (lo, hi) in enumerate(shards):
        lens_s = list(doc_lens[lo:hi])
        for h in range(Hkv):
            kr, chunk_doc = build_routing_keys(R[h, off[lo]:off[hi]], lens_s, chunk)
            for b in range(B):
                qb = block_mean_query(Qr[b, h], route_block)
                for blk in range(nblk):
                    sc = route_doc_scores(qb[blk], kr, chunk_doc, hi - lo)
                    loc = select_top_k(sc, min(top_k, hi - lo))
                    cand_ix[s][b, blk, h] = loc + lo
                    cand_sc[s][b, blk, h] = sc[loc]
    topk = np.empty((B, nblk, Hkv, top_k), dtype=np.int64)
    for b in range(B):
        for blk in range(nblk):
            for h in range(Hkv):
                topk[b, blk, h] = merge_candidates([c[b, blk, h] for c in cand_sc],
                                                   [c[b, blk, h] for c in cand_ix], top_k)[0]

    K_rot = np.empty_like(K)
    for h in range(Hkv):
        K_rot[h] = parallel_rope_bank(K[h], doc_lens, base)
    part_out = np.zeros((n_shards, B, Hq, Tq, d))
    part_lse = np.full((n_shards, B, Hq, Tq), -math.inf)
    out = np.empty((B, Hq, Tq, d))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for t in range(Tq):
                i = Lc - Tq + t
                q_rot = rope(Q[b, hq, t], k_off + i, base)
                docs = topk[b, t // route_block, h]
                for s, (lo, hi) in enumerate(shards):
                    mine = [int(j) for j in docs if lo <= j < hi]
                    ks = [K_rot[h, off[j]:off[j + 1]] for j in mine]
                    vs = [V[h, off[j]:off[j + 1]] for j in mine]
                    if s == owner:
                        ks.append(rope(LK[b, h, :i + 1], k_off + np.arange(i + 1), base))
                        vs.append(LV[b, h, :i + 1])
                    keys = np.concatenate(ks, axis=0) if ks else np.zeros((0, d))
                    vals = np.concatenate(vs, axis=0) if vs else np.zeros((0, d))
                    part_out[s, b, hq, t], part_lse[s, b, hq, t] = attention_partial(q_rot, keys, vals)
                out[b, hq, t] = merge_partials(part_out[:, b, hq, t], part_lse[:, b, hq, t])[0]
    return {"topk": topk, "cand_scores": cand_sc, "cand_idx": cand_ix, "part_out": part_out,
            "part_lse": part_lse, "out": out, "shards": shards, "k_off": k_off}


# --------------------------------------------------------------------------
# Memory Interleave: several hops of routing, each expanding the context
#   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory
#      Interleave: generation of document identifiers and context expansion
#      alternate, so retrieval proceeds in several steps over scattered memory);
#   -- "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §3.2 (several retrieval rounds,
#      each building on the previous one).
# Reading (there is no generating model here, so the "next identifiers" come from
# a stated routing-space update): hop t routes with its routing query q_t over the
# documents not yet in the context, keeps top_k of them and appends them to the
# context; the next hop's query is q_{t+1} = q_t/|q_t| + (1/top_k) sum over the
# hop's documents of kbar_j/|kbar_j|, kbar_j being document j's routing key (the
# mean of its per-token routing keys); after hop t the attention runs over every
# document retrieved so far (t * top_k of them, Global-RoPE offset
# t * top_k * max length) plus the local context.
# --------------------------------------------------------------------------

def doc_routing_key(R_doc: np.ndarray) -> np.ndarray:
    """A document's routing key: the mean of its per-token routing keys [L, d_r]."""
    R_doc = np.asarray(R_doc, dtype=np.float64)
    total = np.zeros(R_doc.shape[1], dtype=np.float64)
    for t in range(R_doc.shape[0]):
        total += R_doc[t]
    return total / R_doc.shape[0]


def interleave_next_query(q_r: np.ndarray, chosen_keys: Sequence[np.ndarray]) -> np.ndarray:
    """The next hop's routing query: q/|q| + (1/k) sum_j kbar_j/|kbar_j| over the hop's k documents."""
    q = np.asarray(q_r, dtype=np.float64)
    out = q / max(math.sqrt(float(q @ q)), 1e-30)
    for kb in chosen_keys:
        kb = np.asarray(kb, dtype=np.float64)
        out = out + kb / max(math.sqrt(float(kb @ kb)), 1e-30) / len(chosen_keys)
    return out


def select_top_k_excluding(doc_scores: np.ndarray, top_k: int, exclude) -> np.ndarray:
    """select_top_k over the documents not in `exclude` (the context already holds them)."""
    s = np.asarray(doc_scores, dtype=np.float64).copy()
    ex = [int(j) for j in exclude]
    if len(s) - len(set(ex)) < top_k:
        raise ValueError("fewer documents outside the context than top_k")
    s[ex] = -np.inf
    return select_top_k(s, top_k)


def memory_interleave(inputs: Dict[str, np.ndarray], doc_lens: Sequence[int], top_k: int, route_block: int,
                      hops: int, base: float = 10000.0, chunk: int = CHUNK) -> Dict[str, list]:
    """Memory Interleave over `hops` hops on explicit inputs (forward()'s layout).

    Per (sequence, routing block, KV head): q_1 = the block mean of the routing
    queries; hop t scores every document (cosine, max over chunks), keeps the top_k
    not yet selected, and forms q_{t+1} = interleave_next_query(q_t, their keys).
    After hop t, each query row attends over all t * top_k documents selected so far
    (hop order, then rank) plus its local context, with k_off = t * top_k * max L.
    Returns per hop: q_r [B, nblk, Hkv, d_r] (the query it routed with), topk
    [B, nblk, Hkv, k] (its new documents), selection [B, nblk, Hkv, t*k] (all so
    far), out [B, Hq, Tq, d]."""
    R = np.asarray(inputs["R"], dtype=np.float64)
    Qr = np.asarray(inputs["Qr"], dtype=np.float64)
    Hkv = R.shape[0]
    B, _, Tq, dr = Qr.shape
    nblk = Tq // route_block
    n = len(doc_lens)
    off = doc_offsets(doc_lens)
    K_r, chunk_doc = [], None
    for h in range(Hkv):
        kr, chunk_doc = build_routing_keys(R[h], doc_lens, chunk)
        K_r.append(kr)
    dkeys = np.stack([np.stack([doc_routing_key(R[h, off[j]:off[j + 1]]) for j in range(n)])
                      for h in range(Hkv)])
    q = np.empty((B, nblk, Hkv, dr))
    for b in range(B):
        for h in range(Hkv):
            q[b, :, h] = block_mean_query(Qr[b, h], route_block)
    res = {"q_r": [], "topk": [], "selection": [], "out": []}
    sel = np.zeros((B, nblk, Hkv, 0), dtype=np.int64)
    for t in range(hops):
        new = np.empty((B, nblk, Hkv, top_k), dtype=np.int64)
        nxt = np.empty_like(q)
        for b in range(B):
            for blk in range(nblk):
                for h in range(Hkv):
                    sc = route_doc_scores(q[b, blk, h], K_r[h], chunk_doc, n)
                    new[b, blk, h] = select_top_k_excluding(sc, top_k, sel[b, blk, h])
                    nxt[b, blk, h] = interleave_next_query(q[b, blk, h], [dkeys[h, j] for j in new[b, blk, h]])
        sel = np.concatenate([sel, new], axis=-1)
        out = forward(inputs, doc_lens, sel.shape[-1], route_block, base, chunk, selection=sel)["out"]
        res["q_r"].append(q.copy())
        res["topk"].append(new)
        res["selection"].append(sel.copy())
        res["out"].append(out)
        q = nxt
    return res
