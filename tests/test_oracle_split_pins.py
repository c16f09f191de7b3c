"""Pins of the fp64 per-split partial oracle (the KV chunks of the
context-parallel forward, RL-Kernel PR #284 "feat(attention): add CP backward
drift validation", Changes: KV chunk size, fixed global_block_index merge
order): its definition checked against the pinned whole-context oracle."""
import math

import torch

import oracle
from paged_kv_decode_31_b200 import inputs as I


def _fold(m, l, acc):
    """Ascending fold of the splits (natural-log units) -> (out, lse)."""
    n = m.shape[-1]
    M = torch.full(m.shape[:-1], -math.inf, dtype=torch.float64)
    L = torch.zeros_like(M)
    A = torch.zeros(acc.shape[:-2] + acc.shape[-1:], dtype=torch.float64)
    for s in range(n):
        ms = m[..., s]
        Mn = torch.maximum(M, ms)
        ok = torch.isfinite(Mn)
        ca = torch.where(ok & torch.isfinite(M), torch.exp(M - Mn), torch.zeros_like(M))
        cs = torch.where(ok & torch.isfinite(ms), torch.exp(ms - Mn), torch.zeros_like(M))
        L = L * ca + l[..., s] * cs
        A = A * ca[..., None] + acc[..., s, :] * cs[..., None]
        M = torch.where(ok, Mn, M)
    out = torch.where(L[..., None] > 0, A / L.clamp_min(1e-300)[..., None], torch.zeros_like(A))
    lse = torch.where(L > 0, M + torch.log(L.clamp_min(1e-300)), torch.full_like(M, -math.inf))
    return out, lse


def test_folding_all_splits_gives_the_whole_context_result():
    di = I.p2_case(2, 5, 700, 8, 2, 64, 16, causal=True, seed=71, seqlens=[700, 130])
    m, l, acc = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                      di.scale, True, 0, 6, split_tokens=128)
    out, lse = _fold(m, l, acc)
    ro, rl = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                               di.scale, True)
    assert torch.allclose(out, ro, atol=1e-12, rtol=0)
    assert torch.allclose(lse.permute(0, 2, 1), rl, atol=1e-12, rtol=0)


def test_one_split_covering_the_context_is_the_unnormalised_attention():
    di = I.p2_case(1, 3, 90, 4, 2, 64, 16, causal=False, seed=72, seqlens=[90])
    m, l, acc = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                      di.scale, False, 0, 1)
    ro, rl = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                               di.scale, False)
    assert torch.allclose(acc[..., 0, :] / l[..., 0:1], ro, atol=1e-12, rtol=0)
    assert torch.allclose((m[..., 0] + torch.log(l[..., 0])).permute(0, 2, 1), rl, atol=1e-12)


def test_splits_a_row_does_not_reach_are_empty():
    di = I.p2_case(1, 2, 300, 4, 2, 64, 16, causal=True, seed=73, seqlens=[150])
    m, l, acc = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                      di.scale, True, 1, 3, split_tokens=64)
    # absolute splits 1..3 = keys [64, 256); context 150: split 3 (keys 192..255) is empty
    assert torch.isneginf(m[..., 2]).all() and (l[..., 2] == 0).all() and (acc[..., 2, :] == 0).all()
    assert torch.isfinite(m[..., 0]).all() and (l[..., 0] > 0).all()
