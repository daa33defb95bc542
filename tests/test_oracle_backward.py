"""Pins of the oracle's backward (CPU, fp64): the gradients of L = sum(d_out * out)
with the selection held fixed, checked against central finite differences, against
torch autograd through one dense SDPA call when every document is selected, and
against the closed form sum of value gradients = sum of d_out."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from tests.test_oracle_pins import _small_inputs


def _loss(inp, lens, top_k, route_block, d_out, sel):
    return float((O.forward(inp, lens, top_k, route_block, selection=sel)["out"] * d_out).sum())


def test_gradients_match_central_differences():
    r = np.random.default_rng(11)
    lens = [3, 5, 2]
    d = 4
    inp, _ = _small_inputs(B=1, Hq=2, Hkv=1, d=d, lens=lens, Lc=6, Tq=3, seed=3)
    top_k, bq = 2, 1
    d_out = r.standard_normal(inp["Q"].shape)
    g = O.backward(inp, lens, top_k, bq, d_out)
    sel = g["selection"]
    eps = 1e-6
    for name, grad in (("Q", "dQ"), ("K", "dK"), ("V", "dV"), ("LK", "dLK"), ("LV", "dLV")):
        num = np.zeros_like(inp[name])
        for ix in np.ndindex(inp[name].shape):
            plus, minus = dict(inp), dict(inp)
            plus[name] = inp[name].copy()
            minus[name] = inp[name].copy()
            plus[name][ix] += eps
            minus[name][ix] -= eps
            num[ix] = (_loss(plus, lens, top_k, bq, d_out, sel) - _loss(minus, lens, top_k, bq, d_out, sel)) / (2 * eps)
        np.testing.assert_allclose(g[grad], num, atol=2e-8, err_msg=name)


def test_all_documents_selected_equals_dense_autograd():
    lens = (30, 17, 44, 9)
    inp, lens = _small_inputs(B=2, Hq=4, Hkv=2, d=8, lens=lens, Lc=7, Tq=3, seed=5)
    n = len(lens)
    d_out = np.random.default_rng(2).standard_normal(inp["Q"].shape)
    g = O.backward(inp, lens, n, 1, d_out)
    leaves = {x: torch.tensor(inp[x], requires_grad=True) for x in ("K", "V", "Q", "LK", "LV")}
    k_off = n * max(lens)
    # one dense SDPA over the whole bank plus the causal local context, positions
    # written out here independently, differentiated by torch autograd (fp64)
    K, V, Q, LK, LV = (leaves[x] for x in ("K", "V", "Q", "LK", "LV"))
    Hkv, N, d = K.shape
    B, Hq, Tq, _ = Q.shape
    Lc = LK.shape[2]
    G = Hq // Hkv
    inv = 10000.0 ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)

    def turn(x, pos):
        ang = pos[..., None] * inv
        c, s = torch.cos(ang), torch.sin(ang)
        a, b = x[..., : d // 2], x[..., d // 2:]
        return torch.cat([a * c - b * s, b * c + a * s], dim=-1)

    doc_pos = torch.cat([torch.arange(L, dtype=torch.float64) for L in lens])
    loc_pos = k_off + torch.arange(Lc, dtype=torch.float64)
    keys = torch.cat([turn(K, doc_pos).unsqueeze(0).expand(B, -1, -1, -1), turn(LK, loc_pos)], 2)
    vals = torch.cat([V.unsqueeze(0).expand(B, -1, -1, -1), LV], 2)
    keys = keys.repeat_interleave(G, dim=1)
    vals = vals.repeat_interleave(G, dim=1)
    qi = Lc - Tq + torch.arange(Tq)
    q = turn(Q, (k_off + qi).to(torch.float64))
    mask = torch.cat([torch.ones(Tq, N, dtype=torch.bool), torch.arange(Lc)[None, :] <= qi[:, None]], dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, keys, vals, attn_mask=mask)
    (ref * torch.from_numpy(d_out)).sum().backward()
    np.testing.assert_allclose(g["out"], ref.detach().numpy(), rtol=1e-10, atol=1e-12)
    for x, grad in (("Q", "dQ"), ("K", "dK"), ("V", "dV"), ("LK", "dLK"), ("LV", "dLV")):
        np.testing.assert_allclose(g[grad], leaves[x].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=x)


def test_value_gradients_sum_to_the_output_gradients():
    """Every row's softmax weights sum to 1, so summed over all keys a row's
    value gradients add up to its d_out: per KV head, the bank and local value
    gradients together equal the sum of d_out over the head's query rows."""
    inp, lens = _small_inputs(B=2, Hq=6, Hkv=3, d=8, lens=(21, 9, 33, 14, 40), Lc=9, Tq=4, seed=8)
    d_out = np.random.default_rng(4).standard_normal(inp["Q"].shape)
    g = O.backward(inp, lens, 3, 2, d_out)
    G = 2
    for h in range(3):
        lhs = g["dV"][h].sum(axis=0) + g["dLV"][:, h].sum(axis=(0, 1))
        rhs = d_out[:, h * G:(h + 1) * G].sum(axis=(0, 1, 2))
        np.testing.assert_allclose(lhs, rhs, atol=1e-11)


def test_rope_adjoint_is_the_transpose():
    r = np.random.default_rng(9)
    x, y = r.standard_normal((5, 8)), r.standard_normal((5, 8))
    pos = np.array([0, 3, 17, 1000, 65541])
    # <R x, y> = <x, R^T y>
    np.testing.assert_allclose((O.rope(x, pos, 10000.0) * y).sum(), (x * O.rope_adjoint(y, pos, 10000.0)).sum(),
                               rtol=1e-12)
