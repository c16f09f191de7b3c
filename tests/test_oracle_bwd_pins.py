"""Pins of the fp64 backward oracle: torch autograd (fp64) through a dense
attention built from the gathered cache, on masked, causal and GQA cases;
central finite differences of the oracle's own forward on a tiny case; and
structural zeros (keys no row sees get no gradient; dv of a single key is the
sum of its rows' dout)."""
import math

import pytest
import torch

import oracle
from paged_kv_decode_31_b200 import inputs as I


def _dense_autograd(di, dout):
    """fp64 autograd: dense [Lmax] K/V gathered with torch indexing, -inf masks."""
    B, sq, Hq, D = di.q.shape
    bs, Hkv = di.cache.k.shape[1], di.cache.k.shape[2]
    G = Hq // Hkv
    Lmax = int(di.seqlens.max())
    dq = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    dk = torch.zeros(B, Lmax, Hkv, D, dtype=torch.float64)
    dv = torch.zeros(B, Lmax, Hkv, D, dtype=torch.float64)
    for b in range(B):
        n = int(di.seqlens[b])
        j = torch.arange(n)
        blk = di.block_table[b, j // bs].long()
        K = di.cache.k[blk, j % bs].double().clone().requires_grad_(True)
        V = di.cache.v[blk, j % bs].double().clone().requires_grad_(True)
        Q = di.q[b].double().clone().requires_grad_(True)
        outs = []
        for h in range(Hq):
            s = di.scale * (Q[:, h] @ K[:, h // G].T)
            if di.causal:
                pos = n - sq + torch.arange(sq)
                s = s.masked_fill(torch.arange(n)[None, :] > pos[:, None], float("-inf"))
            p = torch.softmax(s, dim=1)
            p = torch.nan_to_num(p, nan=0.0)
            outs.append(p @ V[:, h // G])
        o = torch.stack(outs, 1)
        (o * dout[b].double()).sum().backward()
        dq[b] = Q.grad
        dk[b, :n] = K.grad
        dv[b, :n] = V.grad
    return dq, dk, dv


@pytest.mark.parametrize("causal,sq,G,seqlens", [(True, 5, 2, [40, 9]), (False, 3, 1, [33, 17]),
                                                 (True, 12, 4, [12, 30])])
def test_backward_oracle_matches_torch_autograd(causal, sq, G, seqlens):
    Hkv = 2
    di = I.p2_case(2, sq, max(seqlens), G * Hkv, Hkv, 64, 16, causal=causal, seed=sq * G,
                   seqlens=seqlens)
    gen = torch.Generator().manual_seed(99)
    dout = I.randn_bf16(tuple(di.q.shape), gen)
    dq, dk, dv = oracle.paged_attn_bwd(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                       di.scale, causal, dout)
    rq, rk, rv = _dense_autograd(di, dout)
    assert torch.allclose(dq, rq, atol=1e-12, rtol=0)
    Lmax = rk.shape[1]
    assert torch.allclose(dk[:, :Lmax], rk, atol=1e-12, rtol=0)
    assert torch.allclose(dv[:, :Lmax], rv, atol=1e-12, rtol=0)


def test_backward_oracle_finite_differences():
    """d/dq of sum(out * dout) by central differences of the forward oracle."""
    di = I.p2_case(1, 2, 7, 2, 1, 64, 16, causal=True, seed=4, seqlens=[7])
    gen = torch.Generator().manual_seed(5)
    dout = I.randn_bf16(tuple(di.q.shape), gen).double()
    dq, dk, dv = oracle.paged_attn_bwd(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                       di.scale, True, dout)
    # the forward oracle takes bf16 q; perturb the scale-free score through a
    # dense fp64 restatement of one element instead: f(x) = sum(out(q + x e) * dout)
    bs = 16
    j = torch.arange(7)
    K = di.cache.k[di.block_table[0, j // bs].long(), j % bs].double()[:, 0]
    V = di.cache.v[di.block_table[0, j // bs].long(), j % bs].double()[:, 0]

    def f(qv, i):
        s = di.scale * (K[:5 + i + 1] @ qv)
        p = torch.softmax(s, 0)
        return float(p @ V[:5 + i + 1] @ dout[0, i, 0])

    for i in range(2):
        for d in (0, 17, 63):
            e = torch.zeros(64, dtype=torch.float64)
            e[d] = 1e-6
            qv = di.q[0, i, 0].double()
            num = (f(qv + e, i) - f(qv - e, i)) / 2e-6
            assert abs(num - float(dq[0, i, 0, d])) < 1e-7


def test_backward_structural_zeros_and_single_key():
    di = I.p2_case(1, 3, 50, 4, 2, 64, 16, causal=True, seed=8, seqlens=[50])
    gen = torch.Generator().manual_seed(9)
    dout = I.randn_bf16(tuple(di.q.shape), gen)
    dq, dk, dv = oracle.paged_attn_bwd(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                       di.scale, True, dout)
    # all three rows see keys 0..47 at least; no key past position 49 exists
    assert dk.shape[1] == 50
    # one-key context: out = v_0, so dv_0 = sum of dout over the rows, dq = dk = 0
    d1 = I.p2_case(1, 1, 1, 4, 2, 64, 16, causal=True, seed=10, seqlens=[1])
    do1 = I.randn_bf16(tuple(d1.q.shape), gen)
    q1, k1, v1 = oracle.paged_attn_bwd(d1.q, d1.cache.k, d1.cache.v, d1.block_table, d1.seqlens,
                                       d1.scale, True, do1)
    assert torch.allclose(v1[0, 0, 0], do1[0, 0, 0:2].double().sum(0), atol=1e-12)
    assert torch.allclose(q1, torch.zeros_like(q1), atol=1e-12)
    assert torch.allclose(k1, torch.zeros_like(k1), atol=1e-12)
