"""Pins of the packed (varlen) oracle functions, independent of the C oracle
they call: a pure-Python fp64 brute force of the packing and of each
request's bottom-right query positions; equal lengths equal the dense call;
a request's rows do not depend on the other requests; empty requests; the
final rows are the rows at cu[b+1] - 1; the packed append places each
request's tokens at seqlens[b] + t.  Source of the packed form: the AstrAI
commit search page ("Pack prompts ... into one forward", "Select per-request
final logits from cumulative query lengths")."""
import math

import torch

import oracle
from paged_kv_decode_31_b200 import inputs as I


def _brute_force(q, k_view, v_view, table, seqlens, cu, scale, causal, Hkv):
    """Plain Python loops in fp64: gather token j of request b from block
    table[b][j // bs], slot j % bs; query i of request b sits at position
    seqlens[b] - n_b + i."""
    total_q, Hq, D = q.shape
    bs = k_view.shape[1]
    G = Hq // Hkv
    out = torch.zeros(total_q, Hq, D, dtype=torch.float64)
    lse = torch.zeros(Hq, total_q, dtype=torch.float64)
    qd, kd, vd = q.double(), k_view.double(), v_view.double()
    for b in range(len(cu) - 1):
        n_b, L = cu[b + 1] - cu[b], int(seqlens[b])
        for i in range(n_b):
            pos = L - n_b + i
            for h in range(Hq):
                g = h // G
                keys = range(min(L, pos + 1) if causal else L)
                if len(keys) == 0:
                    lse[h, cu[b] + i] = -math.inf
                    continue
                s = []
                for j in keys:
                    blk = int(table[b, j // bs])
                    s.append(scale * float(qd[cu[b] + i, h] @ kd[blk, j % bs, g]))
                m = max(s)
                w = [math.exp(x - m) for x in s]
                l = sum(w)
                acc = torch.zeros(D, dtype=torch.float64)
                for wj, j in zip(w, keys):
                    blk = int(table[b, j // bs])
                    acc += wj * vd[blk, j % bs, g]
                out[cu[b] + i, h] = acc / l
                lse[h, cu[b] + i] = m + math.log(l)
    return out, lse


def _case(lengths, ctx, causal, seed=0):
    B = len(ctx)
    di = I.p2_case(B, 1, max(ctx), 4, 2, 16 * 4, 16, causal=causal, seed=seed, seqlens=ctx)
    gen = torch.Generator().manual_seed(seed + 1)
    total = sum(lengths)
    q = I.randn_bf16((total, 4, 64), gen)
    cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()), dtype=torch.int32)
    return di, q, cu


def test_varlen_oracle_matches_python_brute_force():
    lengths, ctx = [3, 0, 1, 5], [40, 17, 9, 4]   # request 3 has more queries than keys
    for causal in (True, False):
        di, q, cu = _case(lengths, ctx, causal, seed=3)
        o, l, fo, fl = oracle.paged_attn_varlen(q, di.cache.k, di.cache.v, di.block_table,
                                                di.seqlens, cu, di.scale, causal)
        ro, rl = _brute_force(q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                              cu.tolist(), di.scale, causal, 2)
        assert torch.allclose(o, ro, atol=1e-12, rtol=0)
        fin = torch.isfinite(rl)
        assert torch.equal(torch.isneginf(l), torch.isneginf(rl))
        assert torch.allclose(l[fin], rl[fin], atol=1e-12, rtol=0)


def test_equal_lengths_equal_the_dense_call():
    di = I.p2_case(3, 6, 500, 8, 2, 128, 16, causal=True, seed=5, seqlens=[500, 321, 7])
    cu = torch.arange(0, 19, 6, dtype=torch.int32)
    o, l, _, _ = oracle.paged_attn_varlen(di.q.reshape(18, 8, 128), di.cache.k, di.cache.v,
                                          di.block_table, di.seqlens, cu, di.scale, True)
    od, ld = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                               di.scale, True)
    assert torch.equal(o.reshape(3, 6, 8, 128), od)
    assert torch.equal(l.reshape(8, 3, 6).permute(1, 0, 2), ld)


def test_requests_are_independent_and_final_rows_are_the_last_rows():
    lengths, ctx = [4, 2, 7], [100, 60, 30]
    di, q, cu = _case(lengths, ctx, True, seed=7)
    o, l, fo, fl = oracle.paged_attn_varlen(q, di.cache.k, di.cache.v, di.block_table,
                                            di.seqlens, cu, di.scale, True)
    for b in range(3):
        a, e = int(cu[b]), int(cu[b + 1])
        assert torch.equal(fo[b], o[e - 1]) and torch.equal(fl[b], l[:, e - 1])
    # request 1 alone (a batch of one) gives the same rows
    o1, l1, _, _ = oracle.paged_attn_varlen(
        q[4:6], di.cache.k, di.cache.v, di.block_table[1:2], di.seqlens[1:2],
        torch.tensor([0, 2], dtype=torch.int32), di.scale, True)
    assert torch.equal(o1, o[4:6]) and torch.equal(l1, l[:, 4:6])


def test_varlen_append_places_tokens_at_seqlen_positions():
    gen = torch.Generator().manual_seed(11)
    di = I.p2_case(3, 1, 200, 4, 2, 64, 16, causal=False, seed=9)
    cache = di.cache.clone()
    before = torch.tensor([0, 50, 17], dtype=torch.int32)
    cu = torch.tensor([0, 3, 3, 8], dtype=torch.int32)   # request 1 appends nothing
    kn = I.randn_bf16((8, 2, 64), gen)
    vn = I.randn_bf16((8, 2, 64), gen)
    oracle.kv_append_varlen(kn, vn, cache.k, cache.v, di.block_table, before, cu)
    bs = 16
    for b, (a, e) in enumerate([(0, 3), (3, 3), (3, 8)]):
        for t in range(e - a):
            p = int(before[b]) + t
            blk = int(di.block_table[b, p // bs])
            assert torch.equal(cache.k[blk, p % bs].view(torch.int16), kn[a + t].view(torch.int16))
            assert torch.equal(cache.v[blk, p % bs].view(torch.int16), vn[a + t].view(torch.int16))
    # nothing else changed
    changed = sum(int((c1.view(torch.int16) != c0.view(torch.int16)).any(-1).any(-1).sum())
                  for c1, c0 in ((cache.k, di.cache.k), (cache.v, di.cache.v)))
    assert changed <= 2 * 8
