"""Packed multi-request attention (pkv_paged_varlen_attn) and the packed
append (pkv_kv_append_varlen) on the GPU: parity with the oracle, each
request's rows bitwise equal to the dense call on that request alone, the
final rows bitwise equal to the last rows, and the query-count bound flag.
Request mixes follow a packed forward of decode steps, multi-token steps and
prefill chunks (AstrAI commit search page: packed prompts, per-request final
rows from cumulative query lengths)."""
import pytest
import torch

import oracle
import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal

pytestmark = pytest.mark.gpu


def _packed(lengths, ctx, Hq, Hkv, D, bs, causal, layout, seed):
    B = len(ctx)
    di = I.p2_case(B, 1, max(ctx), Hq, Hkv, D, bs, causal=causal, layout=layout, seed=seed,
                   seqlens=ctx, poison=True)
    gen = torch.Generator().manual_seed(seed + 17)
    q = I.randn_bf16((sum(lengths), Hq, D), gen)
    cu = torch.tensor([0] + torch.tensor(lengths).cumsum(0).tolist(), dtype=torch.int32)
    return di, q, cu


def _run(di, q, cu, max_q, causal, err=None):
    d = di.to("cuda")
    e = err if err is not None else torch.zeros(1, dtype=torch.int32, device="cuda")
    res = pkv.paged_varlen_attn(q.cuda(), d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                cu.cuda(), max_q, scale=di.scale, causal=causal, final=True,
                                err=e)
    torch.cuda.synchronize()
    if err is None:
        assert int(e.item()) == 0
    return tuple(t.cpu() for t in res)


MIXES = [
    # (query lengths, contexts)
    ([1, 0, 17, 300, 64, 5], [5000, 100, 4500, 9000, 64, 20]),   # 20 < ... rows without keys
    ([1, 1, 1, 1, 3, 2], [131, 4096, 4097, 1, 700, 2]),          # decode-sized: transposed kernel
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mix", range(len(MIXES)))
def test_varlen_matches_oracle(mix, d, causal):
    lengths, ctx = MIXES[mix]
    di, q, cu = _packed(lengths, ctx, 16, 4, d, 16, causal, "interleaved", seed=mix * 10 + d)
    out, lse, fo, fl = _run(di, q, cu, max(lengths), causal)
    ro, rl, rfo, rfl = oracle.paged_attn_varlen(q, di.cache.k, di.cache.v, di.block_table,
                                                di.seqlens, cu, di.scale, causal)
    assert_close_to_oracle(out.unsqueeze(0), lse.unsqueeze(0), ro.unsqueeze(0), rl.unsqueeze(0))
    has = [b for b in range(len(lengths)) if lengths[b] > 0]
    assert_close_to_oracle(fo[has].unsqueeze(1), fl[has].unsqueeze(-1),
                           rfo[has].unsqueeze(1), rfl[has].unsqueeze(-1))


@pytest.mark.parametrize("mix", range(len(MIXES)))
def test_varlen_rows_equal_the_dense_call_bitwise(mix):
    lengths, ctx = MIXES[mix]
    di, q, cu = _packed(lengths, ctx, 16, 4, 128, 32, True, "contiguous", seed=90 + mix)
    out, lse, fo, fl = _run(di, q, cu, max(lengths), True)
    d = di.to("cuda")
    for b, n in enumerate(lengths):
        if n == 0:
            continue
        a = int(cu[b])
        o_b, l_b = pkv.paged_decode_attn(q[a:a + n].unsqueeze(0).cuda(), d.cache.k, d.cache.v,
                                         d.block_table[b:b + 1], d.seqlens[b:b + 1],
                                         max_seqlen_k=ctx[b], scale=di.scale, causal=True)
        torch.cuda.synchronize()
        assert bits_equal(o_b[0].cpu(), out[a:a + n]), f"request {b} out"
        assert bits_equal(l_b[0].cpu(), lse[:, a:a + n]), f"request {b} lse"
        assert bits_equal(fo[b], out[a + n - 1]) and bits_equal(fl[b], lse[:, a + n - 1])


def test_varlen_query_count_above_the_bound_is_flagged():
    lengths, ctx = [2, 9, 1], [300, 300, 300]
    di, q, cu = _packed(lengths, ctx, 8, 2, 128, 16, True, "contiguous", seed=5)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, fo, fl = _run(di, q, cu, 4, True, err=err)     # request 1 has 9 > 4
    assert int(err.item()) & pkv.binding.DEVERR_QUERY_LEN
    ro, rl, _, _ = oracle.paged_attn_varlen(q, di.cache.k, di.cache.v, di.block_table,
                                            di.seqlens, cu, di.scale, True)
    # requests within the bound are still right
    for a, e in ((0, 2), (11, 12)):
        assert_close_to_oracle(out[a:e].unsqueeze(0), lse[:, a:e].unsqueeze(0),
                               ro[a:e].unsqueeze(0), rl[:, a:e].unsqueeze(0))


@pytest.mark.parametrize("layout", ["contiguous", "interleaved"])
def test_kv_append_varlen_matches_oracle_bits(layout):
    gen = torch.Generator().manual_seed(77)
    di = I.p2_case(4, 1, 3000, 8, 4, 128, 16, causal=False, layout=layout, seed=78)
    before = torch.tensor([0, 100, 1400, 7], dtype=torch.int32)
    lengths = [5, 0, 512, 1]
    cu = torch.tensor([0] + torch.tensor(lengths).cumsum(0).tolist(), dtype=torch.int32)
    kn = I.randn_bf16((sum(lengths), 4, 128), gen)
    vn = I.randn_bf16((sum(lengths), 4, 128), gen)
    ref = di.cache.clone()
    oracle.kv_append_varlen(kn, vn, ref.k, ref.v, di.block_table, before, cu)
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_append_varlen(kn.cuda(), vn.cuda(), d.cache.k, d.cache.v, d.block_table,
                         before.cuda(), cu.cuda(), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for g, r in zip(d.cache.backing, ref.backing):
        assert bits_equal(g.cpu(), r)
