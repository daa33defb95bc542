"""Device-resident synthetic inputs (torch allocates, libmsasynth.so fills).

Same values as the numpy generator in synth/__init__.py, bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (NORMAL_TABLE_BITS, T_K, T_LK, T_LV, T_Q, T_QR, T_R, T_V, Workload, device_normal_bf16,
               f32_tensor, planted_qr_bits)

_TABLES = {}


def _table(device) -> torch.Tensor:
    key = str(device)
    if key not in _TABLES:
        _TABLES[key] = torch.from_numpy(NORMAL_TABLE_BITS.view(np.int16).copy()).to(device)
    return _TABLES[key]


def fill_normal(t: torch.Tensor, seed: int, tensor_id: int, start: int = 0) -> torch.Tensor:
    """Fill a contiguous bf16 CUDA tensor with elements [start, start + numel) of a stream."""
    assert t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous()
    device_normal_bf16(t.data_ptr(), seed, tensor_id, start, t.numel(), _table(t.device).data_ptr(),
                       torch.cuda.current_stream(t.device).cuda_stream)
    return t


def normal(shape, seed: int, tensor_id: int, device="cuda", start: int = 0) -> torch.Tensor:
    return fill_normal(torch.empty(shape, dtype=torch.bfloat16, device=device), seed, tensor_id, start)


def _f32(w: Workload, tensor_id: int, shape, device) -> torch.Tensor:
    return torch.from_numpy(f32_tensor(w, tensor_id, shape)).to(device)


def bank_tensors(w: Workload, device="cuda", with_r: bool = True):
    """K, V as [Hkv, kv_rows, d] and R as [Hkv, Ntok, d_r], bf16 (K without RoPE);
    fp32 for an fp32 workload (generated on the host, copied)."""
    shape = (w.n_kv_heads, w.kv_rows, w.head_dim)
    if w.dtype == "f32":
        assert not w.kv_slabs and not w.planted
        R = _f32(w, T_R, (w.n_kv_heads, w.n_tokens, w.route_dim), device) if with_r else None
        return _f32(w, T_K, shape, device), _f32(w, T_V, shape, device), R
    K = normal(shape, w.seed, T_K, device)
    V = normal(shape, w.seed, T_V, device)
    R = normal((w.n_kv_heads, w.n_tokens, w.route_dim), w.seed, T_R, device) if with_r else None
    return K, V, R


def query_tensors(w: Workload, device="cuda"):
    """Q [B,Hq,Tq,d], Qr [B,Hkv,Tq,d_r], local K/V [B,Hkv,Lc,d], all bf16 (fp32 for an fp32 workload)."""
    if w.dtype == "f32":
        return (_f32(w, T_Q, (w.batch, w.n_q_heads, w.q_tokens, w.head_dim), device),
                _f32(w, T_QR, (w.batch, w.n_kv_heads, w.q_tokens, w.route_dim), device),
                _f32(w, T_LK, (w.batch, w.n_kv_heads, w.local_len, w.head_dim), device),
                _f32(w, T_LV, (w.batch, w.n_kv_heads, w.local_len, w.head_dim), device))
    Q = normal((w.batch, w.n_q_heads, w.q_tokens, w.head_dim), w.seed, T_Q, device)
    if w.planted:
        bits = planted_qr_bits(w)
        Qr = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device).contiguous()
    else:
        Qr = normal((w.batch, w.n_kv_heads, w.q_tokens, w.route_dim), w.seed, T_QR, device)
    LK = normal((w.batch, w.n_kv_heads, w.local_len, w.head_dim), w.seed, T_LK, device)
    LV = normal((w.batch, w.n_kv_heads, w.local_len, w.head_dim), w.seed, T_LV, device)
    return Q, Qr, LK, LV


def host_kv_pool(w: Workload, device="cuda"):
    """The pinned-host K/V tier of an aliased bank: [Hkv, kv_slabs * max_len, d] bf16
    in pinned host memory, K with Parallel RoPE (slab rows at positions 0..max_len-1,
    so every document reading the first L_j rows of a slab sees positions 0..L_j-1).
    The RoPE runs on the device through a bank whose documents are the slabs."""
    from sparse_attention_routed_b200.runner import Bank
    assert w.kv_slabs > 0
    K, V, _ = bank_tensors(w, device, with_r=False)
    slabs = Bank(K, V, [w.max_len] * w.kv_slabs, w.rope_base)
    slabs.build(None)
    torch.cuda.synchronize()
    slabs.close()
    Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    Kh.copy_(K)
    Vh.copy_(V)
    del K, V
    torch.cuda.empty_cache()
    return Kh, Vh
