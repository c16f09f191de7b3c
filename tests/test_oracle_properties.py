"""Property-based pins of the oracle (hypothesis): on randomly drawn small
problems -- any batch, query count, group size, head_dim, block size, context
length (zero included), causal or not, contiguous or K/V-interleaved cache,
shuffled block tables with spare blocks -- oracle.paged_attn equals the plain
definition of paged attention (gather the context through the block table,
softmax(scale q K^T) V, lse = log-sum-exp), written here independently with
torch fp64 ops, and oracle.kv_append places every token at its position."""
import math

import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SHAPES = st.fixed_dictionaries({
    "B": st.integers(1, 3),
    "sq": st.integers(1, 5),
    "G": st.integers(1, 3),
    "Hkv": st.integers(1, 2),
    "D": st.sampled_from([4, 8, 16]),
    "bs": st.sampled_from([1, 2, 4, 8]),
    "max_ctx": st.integers(0, 40),
    "causal": st.booleans(),
    "interleaved": st.booleans(),
    "spare": st.integers(0, 5),
    "seed": st.integers(0, 2**31 - 1),
})


def _problem(c):
    g = torch.Generator().manual_seed(c["seed"])
    B, sq, Hkv, D, bs = c["B"], c["sq"], c["Hkv"], c["D"], c["bs"]
    Hq = c["G"] * Hkv
    seqlens = torch.randint(0, c["max_ctx"] + 1, (B,), generator=g, dtype=torch.int32)
    width = max(1, math.ceil(c["max_ctx"] / bs))
    nb = B * width + c["spare"]
    if c["interleaved"]:
        kv = torch.randn(nb, 2, bs, Hkv, D, generator=g).to(torch.bfloat16)
        k, v = kv[:, 0], kv[:, 1]
    else:
        k = torch.randn(nb, bs, Hkv, D, generator=g).to(torch.bfloat16)
        v = torch.randn(nb, bs, Hkv, D, generator=g).to(torch.bfloat16)
    table = torch.randperm(nb, generator=g)[:B * width].to(torch.int32).reshape(B, width)
    q = torch.randn(B, sq, Hq, D, generator=g).to(torch.bfloat16)
    scale = float(torch.empty(()).uniform_(0.05, 1.0, generator=g))
    return q, k, v, table, seqlens, scale


def _definition(q, k, v, table, seqlens, scale, causal):
    B, sq, Hq, D = q.shape
    bs, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    lse = torch.full((B, Hq, sq), -math.inf, dtype=torch.float64)
    for b in range(B):
        n = int(seqlens[b])
        if n == 0:
            continue
        idx = torch.arange(n)
        blk = table[b, idx // bs].long()
        K = k[blk, idx % bs].double()  # [n, Hkv, D]
        V = v[blk, idx % bs].double()
        for i in range(sq):
            lim = min(n, n - sq + i + 1) if causal else n
            if lim <= 0:
                continue
            for h in range(Hq):
                s = scale * (K[:lim, h // G] @ q[b, i, h].double())
                lse[b, h, i] = torch.logsumexp(s, 0)
                out[b, i, h] = torch.softmax(s, 0) @ V[:lim, h // G]
    return out, lse


@settings(max_examples=60, deadline=None)
@given(SHAPES)
def test_oracle_equals_the_definition_on_random_problems(c):
    q, k, v, table, seqlens, scale = _problem(c)
    out, lse = oracle.paged_attn(q, k, v, table, seqlens, scale, c["causal"])
    ref_out, ref_lse = _definition(q, k, v, table, seqlens, scale, c["causal"])
    assert torch.allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(lse), fin)
    assert torch.allclose(lse[fin], ref_lse[fin], rtol=1e-12, atol=1e-12)
    assert torch.all(out[~fin.permute(0, 2, 1)] == 0)  # rows that see no key


@settings(max_examples=40, deadline=None)
@given(SHAPES, st.integers(0, 6))
def test_kv_append_places_every_token_at_its_position(c, n_new):
    q, k, v, table, seqlens, _ = _problem(c)
    B, Hkv, D, bs = q.shape[0], k.shape[2], k.shape[3], k.shape[1]
    cap = table.shape[1] * bs
    before = torch.clamp(seqlens, max=max(cap - n_new, 0))
    if int(before.max()) + n_new > cap:
        return  # this draw has no room for the new tokens
    g = torch.Generator().manual_seed(c["seed"] + 1)
    kn = torch.randn(B, n_new, Hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, n_new, Hkv, D, generator=g).to(torch.bfloat16)
    k0, v0 = k.clone(), v.clone()
    oracle.kv_append(kn, vn, k, v, table, before)
    touched = torch.zeros(k.shape[0], bs, dtype=torch.bool)
    for b in range(B):
        for t in range(n_new):
            p = int(before[b]) + t
            blk, slot = int(table[b, p // bs]), p % bs
            assert torch.equal(k[blk, slot].view(torch.int16), kn[b, t].view(torch.int16))
            assert torch.equal(v[blk, slot].view(torch.int16), vn[b, t].view(torch.int16))
            touched[blk, slot] = True
    # nothing else changed
    assert torch.equal(k[~touched].view(torch.int16), k0[~touched].view(torch.int16))
    assert torch.equal(v[~touched].view(torch.int16), v0[~touched].view(torch.int16))


@settings(max_examples=40, deadline=None)
@given(SHAPES, st.sampled_from([1, 2, 3, 5, 8, 16]), st.integers(1, 4))
def test_rank_shares_of_split_partials_fold_to_the_whole_context(c, split_tokens, world):
    """Context parallelism on the oracle side: the splits cut into `world`
    contiguous shares of ceil(S / world) (the last ones may run past the
    context), each share's partials computed alone, laid side by side and
    folded in ascending split order equal the whole-context result."""
    from test_oracle_split_pins import _fold

    q, k, v, table, seqlens, scale = _problem(c)
    S = max(1, math.ceil(c["max_ctx"] / split_tokens))
    n_local = math.ceil(S / world)
    parts = [oracle.split_partials(q, k, v, table, seqlens, scale, c["causal"], r * n_local,
                                   n_local, split_tokens=split_tokens) for r in range(world)]
    m = torch.cat([p[0] for p in parts], -1)
    l = torch.cat([p[1] for p in parts], -1)
    acc = torch.cat([p[2] for p in parts], -2)
    out, lse = _fold(m, l, acc)
    ref_out, ref_lse = oracle.paged_attn(q, k, v, table, seqlens, scale, c["causal"])
    assert torch.allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    lse = lse.permute(0, 2, 1)
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(lse), fin)
    assert torch.allclose(lse[fin], ref_lse[fin], rtol=1e-12, atol=1e-12)


@settings(max_examples=30, deadline=None)
@given(SHAPES)
def test_backward_oracle_equals_autograd_on_random_problems(c):
    """The fp64 backward oracle against torch autograd through the dense
    definition, on the same random problems (rows that see no key included:
    they get no gradient)."""
    from test_oracle_bwd_pins import _dense_autograd

    from paged_kv_decode_31_b200 import inputs as I

    q, k, v, table, seqlens, scale = _problem(c)
    Hq, Hkv, D = q.shape[2], k.shape[2], q.shape[3]
    layout = "interleaved" if c["interleaved"] else "contiguous"
    cache = I.PagedCache(k, v, (k, v), layout)
    di = I.DecodeInputs(q, cache, table, seqlens, Hq, Hkv, D, scale, c["causal"])
    g = torch.Generator().manual_seed(c["seed"] + 2)
    dout = torch.randn(tuple(q.shape), generator=g).to(torch.bfloat16)
    dq, dk, dv = oracle.paged_attn_bwd(q, k, v, table, seqlens, scale, c["causal"], dout)
    rq, rk, rv = _dense_autograd(di, dout)
    assert torch.allclose(dq, rq, rtol=1e-12, atol=1e-12)
    L = rk.shape[1]
    assert torch.allclose(dk[:, :L], rk, rtol=1e-12, atol=1e-12)
    assert torch.allclose(dv[:, :L], rv, rtol=1e-12, atol=1e-12)
    assert not (dk[:, L:].any() or dv[:, L:].any())


@settings(max_examples=40, deadline=None)
@given(SHAPES, st.lists(st.integers(0, 6), min_size=3, max_size=3))
def test_packed_oracle_equals_each_request_alone(c, n_q):
    """Packed queries: request b's n_b rows (rows cu[b] .. cu[b+1]-1 of the
    packed q) are the last n_b positions of its context; each request's rows
    equal the plain definition on that request alone, lse is [Hq, total_q],
    and the final rows are the rows at cu[b+1]-1."""
    q, k, v, table, seqlens, scale = _problem(c)
    B, Hq, D = q.shape[0], q.shape[2], q.shape[3]
    n_q = n_q[:B]
    if sum(n_q) == 0:
        n_q[0] = 1
    g = torch.Generator().manual_seed(c["seed"] + 3)
    qp = torch.randn(sum(n_q), Hq, D, generator=g).to(torch.bfloat16)
    cu = torch.tensor([0] + list(torch.tensor(n_q).cumsum(0)), dtype=torch.int32)
    out, lse, fin_out, fin_lse = oracle.paged_attn_varlen(qp, k, v, table, seqlens, cu, scale,
                                                          c["causal"])
    for b in range(B):
        a, e = int(cu[b]), int(cu[b + 1])
        if e == a:
            continue
        ro, rl = _definition(qp[a:e].unsqueeze(0), k, v, table[b:b + 1], seqlens[b:b + 1],
                             scale, c["causal"])
        assert torch.allclose(out[a:e], ro[0], rtol=1e-12, atol=1e-12)
        fin = torch.isfinite(rl[0])
        assert torch.equal(torch.isfinite(lse[:, a:e]), fin)
        assert torch.allclose(lse[:, a:e][fin], rl[0][fin], rtol=1e-12, atol=1e-12)
        assert torch.equal(fin_out[b], out[e - 1])
        assert torch.equal(fin_lse[b], lse[:, e - 1])
