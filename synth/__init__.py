"""Seeded synthetic inputs for the routed sparse-attention step.

This module is shared by the CUDA library's tests/bench and by the CPU oracle's
tests. It holds none of the method's arithmetic: it only draws numbers and
describes workload shapes.

Generator (counter-based, identical on the CPU and on the GPU):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the 64-bit finaliser published with it):
  ``mix64(z)`` = xor-shift-multiply by 0xBF58476D1CE4E5B9 and
  0x94D049BB133111EB with shifts 30, 27, 31.
* Stream key of a tensor: ``key = mix64(seed*GAMMA + tensor_id*GAMMA2 + 1)``.
* Element ``i`` of the tensor (its flat row-major index) draws
  ``u = mix64(key + (i + 1) * GAMMA)``: the i-th output of SplitMix64 started
  at ``key``, so any slice can be regenerated on its own.
* Normal values: ``TABLE[u >> 48]`` where ``TABLE[j]`` is the inverse normal
  CDF at ``(j + 0.5) / 65536`` computed in fp64 and rounded to bfloat16
  (round to nearest even). The values are N(0,1) quantised to 65536 levels
  (|x| <= 4.33) and exactly representable in bf16 and fp32, so "bf16 inputs"
  and "fp32 inputs rounded to bf16" are the same numbers.

The CUDA twin of ``normal_bf16_bits`` is ``synth/synth_gen.cu`` (built into
``synth/libmsasynth.so``); ``tests/test_gpu_synth.py`` checks they agree bit
for bit.
"""
from __future__ import annotations

import ctypes
import math
import os
import statistics
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
GAMMA2 = 0xD1B54A32D192ED03

# tensor ids
T_K, T_V, T_R, T_Q, T_QR, T_LK, T_LV, T_LENS, T_TARGETS, T_Z = range(1, 11)


def _mix64_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.atleast_1d(np.asarray(z, dtype=np.uint64))
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix64_int(seed * GAMMA + tensor_id * GAMMA2 + 1)


def u64_at(key: int, idx) -> np.ndarray:
    """The idx-th (0-based) SplitMix64 output of the stream started at key."""
    scalar = np.ndim(idx) == 0
    idx = np.atleast_1d(np.asarray(idx, dtype=np.uint64))
    with np.errstate(over="ignore"):
        out = mix64(np.uint64(key) + (idx + np.uint64(1)) * np.uint64(GAMMA))
    return out[0] if scalar else out


def _round_f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 value (ties to even), returned as fp64."""
    m, e = np.frexp(x)  # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def _build_table():
    nd = statistics.NormalDist()
    v = np.array([nd.inv_cdf((j + 0.5) / 65536.0) for j in range(65536)], dtype=np.float64)
    v = _round_f64_to_bf16(v).astype(np.float32)
    bits = (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << np.uint32(16)).view(np.float32), v)
    return v, bits


NORMAL_TABLE_F32, NORMAL_TABLE_BITS = _build_table()


def normal_bf16_bits(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """bf16 bit patterns of elements [start, start+count) of a normal tensor."""
    key = stream_key(seed, tensor_id)
    idx = np.arange(start, start + count, dtype=np.uint64)
    return NORMAL_TABLE_BITS[(u64_at(key, idx) >> np.uint64(48)).astype(np.int64)]


def normal_f32(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    key = stream_key(seed, tensor_id)
    idx = np.arange(start, start + count, dtype=np.uint64)
    return NORMAL_TABLE_F32[(u64_at(key, idx) >> np.uint64(48)).astype(np.int64)]


# fp32 workloads draw from streams of their own (tensor id + F32_STREAMS)
F32_STREAMS = 100


def gaussian_f32(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Elements [start, start+count) of an fp32 N(0,1) tensor whose values use all
    24 significant bits (unlike the table values, which are bf16 numbers).

    Element i is the Box-Muller transform (Box & Muller, "A note on the generation
    of random normal deviates", Ann. Math. Statist. 1958) of two 53-bit uniforms,
    outputs 2i and 2i+1 of the tensor's SplitMix64 stream:
    u1 = (top 53 bits + 1) / 2^53 in (0, 1], u2 = top 53 bits / 2^53 in [0, 1),
    z = sqrt(-2 ln u1) cos(2 pi u2), computed in fp64 and rounded to fp32."""
    key = stream_key(seed, tensor_id + F32_STREAMS)
    idx = np.arange(start, start + count, dtype=np.uint64)
    a = u64_at(key, idx * np.uint64(2)) >> np.uint64(11)
    b = u64_at(key, idx * np.uint64(2) + np.uint64(1)) >> np.uint64(11)
    u1 = (a.astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = b.astype(np.float64) * 2.0 ** -53
    return (np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)).astype(np.float32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); finite inputs only."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    seed: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_docs: int
    doc_len: int            # fixed length, or 0 for ragged
    local_len: int
    q_tokens: int
    route_block: int
    top_k: int
    ragged: Optional[tuple] = None   # (lo, hi) inclusive, lengths not multiples of 256
    planted: int = 0                 # planted target docs per sequence
    host_tier: bool = False
    kv_slabs: int = 0                # > 0: K/V of document j are the rows of slab (j mod kv_slabs)
    rope_base: float = 10000.0
    dtype: str = "bf16"              # "f32": fp32 tensors from gaussian_f32 (device-tier banks)
    doc_lens_cache: Optional[np.ndarray] = field(default=None, repr=False)

    @property
    def route_dim(self) -> int:
        return self.head_dim

    def doc_lens(self) -> np.ndarray:
        if self.doc_lens_cache is None:
            if self.ragged is None:
                self.doc_lens_cache = np.full(self.n_docs, self.doc_len, dtype=np.int64)
            else:
                self.doc_lens_cache = ragged_lengths(self.seed, self.n_docs, *self.ragged)
        return self.doc_lens_cache

    @property
    def n_tokens(self) -> int:
        return int(self.doc_lens().sum())

    @property
    def max_len(self) -> int:
        return int(self.doc_lens().max())

    @property
    def kv_rows(self) -> int:
        """Rows per head of the K/V tensors (the slab pool when aliased)."""
        return self.kv_slabs * self.max_len if self.kv_slabs else self.n_tokens

    def doc_kv_rows(self) -> np.ndarray:
        """First K/V row of every document inside each head's K/V tensor."""
        if self.kv_slabs:
            return (np.arange(self.n_docs, dtype=np.int64) % self.kv_slabs) * self.max_len
        return np.concatenate([[0], np.cumsum(self.doc_lens())[:-1]]).astype(np.int64)

    def scaled(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        d["doc_lens_cache"] = None
        return Workload(**d)


def ragged_lengths(seed: int, n_docs: int, lo: int, hi: int) -> np.ndarray:
    """Lengths uniform on [lo, hi]; a multiple of 256 is redrawn from the next counter."""
    key = stream_key(seed, T_LENS)
    span = hi - lo + 1
    out = np.empty(n_docs, dtype=np.int64)
    for j in range(n_docs):
        a = 0
        while True:
            u = int(u64_at(key, j * 64 + a))
            L = lo + u % span
            if L % 256 != 0:
                break
            a += 1
        out[j] = L
    return out


def planted_targets(seed: int, batch: int, n_docs: int, count: int) -> np.ndarray:
    """count distinct target documents per sequence, [batch, count] int64."""
    key = stream_key(seed, T_TARGETS)
    out = np.empty((batch, count), dtype=np.int64)
    for b in range(batch):
        got: List[int] = []
        a = 0
        while len(got) < count:
            j = int(u64_at(key, b * 4096 + a)) % n_docs
            a += 1
            if j not in got:
                got.append(j)
        out[b] = got
    return out


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 4, 4, 64, 16, 512, 256, 16, 16, 2),
    # the tiny step with fp32 values (24 significant bits) and the fp32 path end to end
    "tiny_f32": Workload("tiny_f32", 0, 1, 4, 4, 64, 16, 512, 256, 16, 16, 2, dtype="f32"),
    "decode_4m": Workload("decode_4m", 1, 8, 32, 8, 128, 1024, 4096, 4096, 1, 1, 16),
    # same step as decode_4m on a 128-document bank: identical attention bytes per
    # step, 2 GB of K/V on the device (for hardware-counter captures)
    "decode_512k": Workload("decode_512k", 1, 8, 32, 8, 128, 128, 4096, 4096, 1, 1, 16),
    "prefill": Workload("prefill", 2, 1, 32, 8, 128, 256, 8192, 4096, 4096, 64, 8),
    # the prefill step on a 64-document bank: same work per CTA, 2 GB of K/V (hardware-counter captures)
    "prefill_64docs": Workload("prefill_64docs", 2, 1, 32, 8, 128, 64, 8192, 4096, 4096, 64, 8),
    # the prefill step with 1024-token documents: a document draws as many problems as in
    # prefill (the backward's key tiles see the same rows), 1 GB of K/V (hardware-counter captures)
    "prefill_short_docs": Workload("prefill_short_docs", 2, 1, 32, 8, 128, 256, 1024, 4096, 4096, 64, 8),
    # K/V of these two banks (283 GB, 410 GB) exceed host RAM: the pinned pool holds
    # kv_slabs distinct slabs and document j reads slab j mod kv_slabs (routing keys
    # stay distinct per document; the bytes each step moves over PCIe are unchanged)
    "ragged_planted": Workload("ragged_planted", 3, 4, 64, 8, 128, 8192, 0, 2048, 1, 1, 32,
                               ragged=(512, 16384), planted=4, host_tier=True, kv_slabs=256),
    "bank_100m": Workload("bank_100m", 4, 16, 32, 8, 128, 24414, 4096, 4096, 1, 1, 16,
                          host_tier=True, kv_slabs=1024),
}


# ----------------------------------------------------------------------------
# host-side tensors (numpy); layouts match the C ABI
# ----------------------------------------------------------------------------

def bank_rows_bits(w: Workload, tensor_id: int, head: int, tok0: int, ntok: int) -> np.ndarray:
    """bf16 bits of rows [tok0, tok0+ntok) of head `head` of a [Hkv, Ntok, d] bank tensor
    (the routing keys; K and V too when the bank is not aliased)."""
    d = w.head_dim
    start = (head * w.n_tokens + tok0) * d
    return normal_bf16_bits(w.seed, tensor_id, start, ntok * d).reshape(ntok, d)


def doc_kv_bits(w: Workload, tensor_id: int, head: int, doc: int, t0: int = 0, n=None) -> np.ndarray:
    """bf16 bits of tokens [t0, t0+n) of document `doc` in K (T_K) or V (T_V)."""
    d = w.head_dim
    n = int(w.doc_lens()[doc]) - t0 if n is None else n
    row = int(w.doc_kv_rows()[doc]) + t0
    start = (head * w.kv_rows + row) * d
    return normal_bf16_bits(w.seed, tensor_id, start, n * d).reshape(n, d)


def f32_tensor(w: Workload, tensor_id: int, shape) -> np.ndarray:
    """A whole fp32 tensor of an fp32 workload, flat index order (host)."""
    return gaussian_f32(w.seed, tensor_id, 0, int(np.prod(shape))).reshape(shape)


def query_bits(w: Workload, tensor_id: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return normal_bf16_bits(w.seed, tensor_id, 0, n).reshape(shape)


def planted_qr_bits(w: Workload) -> np.ndarray:
    """Per-token routing queries with planted targets, [B, Hkv, 1, d_r] bf16 bits.

    KV head h of sequence b aims at target t = targets[b, h % planted]:
    q_r = 0.6 * mu/|mu| + 0.4 * z/sqrt(d_r), mu = mean of doc t's routing keys
    for head h (fp64), z ~ N(0, I); then rounded to bf16.
    """
    assert w.q_tokens == 1
    d = w.route_dim
    targets = planted_targets(w.seed, w.batch, w.n_docs, w.planted)
    lens = w.doc_lens()
    off = np.concatenate([[0], np.cumsum(lens)])
    z = normal_f32(w.seed, T_Z, 0, w.batch * w.n_kv_heads * d).astype(np.float64)
    z = z.reshape(w.batch, w.n_kv_heads, d)
    out = np.empty((w.batch, w.n_kv_heads, 1, d), dtype=np.uint16)
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            t = int(targets[b, h % w.planted])
            R = bf16_bits_to_f32(bank_rows_bits(w, T_R, h, int(off[t]), int(lens[t]))).astype(np.float64)
            mu = R.mean(axis=0)
            v = 0.6 * mu / np.linalg.norm(mu) + 0.4 * z[b, h] / math.sqrt(d)
            out[b, h, 0] = f32_to_bf16_bits(v.astype(np.float32))
    return out


# ----------------------------------------------------------------------------
# device twin
# ----------------------------------------------------------------------------

_LIB = None
_TABLE_DEV = {}


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmsasynth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"synthetic-input CUDA library not built: {path}")
        lib = ctypes.CDLL(path)
        lib.synth_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_normal_bf16.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def device_normal_bf16(out_ptr: int, seed: int, tensor_id: int, start: int, count: int,
                       table_ptr: int, stream: int = 0) -> None:
    """Fill `count` bf16 values at device pointer out_ptr with elements [start, start+count)."""
    rc = _lib().synth_normal_bf16(ctypes.c_void_p(out_ptr), stream_key(seed, tensor_id), start,
                                  count, ctypes.c_void_p(table_ptr), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synth_normal_bf16 failed: cuda error {rc}")
