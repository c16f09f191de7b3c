"""Fused append + decode (pkv_paged_decode_attn_append) against the two-call
path kv_append + paged_decode_attn: the cache must hold the same bits and out /
lse must be bitwise equal; and against the oracle (append, then attention).
The aiter test grid exercises flash_attn_with_kvcache with and without new_kv;
this is the new_kv form."""
import pytest
import torch

import oracle
import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal

pytestmark = pytest.mark.gpu

CASES = [
    # (batch, n_new = seqlen_q, context after append, Hq, Hkv, D, bs, layout, causal)
    (4, 1, 5000, 32, 8, 128, 16, "contiguous", False),
    (3, 1, 700, 16, 4, 64, 256, "interleaved", False),
    (2, 3, 4097, 8, 2, 128, 16, "interleaved", True),    # new tokens straddle a split boundary
    (2, 17, 1500, 16, 4, 128, 32, "contiguous", True),    # 68 rows: two row tiles
    (5, 1, 9000, 8, 8, 128, 64, "contiguous", False),     # G = 1
    (2, 200, 3000, 16, 4, 128, 16, "interleaved", True),  # prefill chunk: append launch first
    (3, 40, 6000, 8, 2, 64, 32, "contiguous", True),      # 160 rows, two splits
]


@pytest.mark.parametrize("B,n,ctx,Hq,Hkv,D,bs,layout,causal", CASES)
def test_fused_append_equals_append_then_decode(B, n, ctx, Hq, Hkv, D, bs, layout, causal):
    gen = torch.Generator().manual_seed(ctx + n)
    sls = [ctx - 7 * b for b in range(B)]
    di = I.p2_case(B, n, ctx, Hq, Hkv, D, bs, causal=causal, layout=layout, seed=ctx + B,
                   seqlens=sls, poison=True)
    kn = I.randn_bf16((B, n, Hkv, D), gen)
    vn = I.randn_bf16((B, n, Hkv, D), gen)
    # two-call path
    d1 = di.to("cuda")
    before = (d1.seqlens - n).contiguous()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_append(kn.cuda(), vn.cuda(), d1.cache.k, d1.cache.v, d1.block_table, before, err=err)
    o1, l1 = pkv.paged_decode_attn(d1.q, d1.cache.k, d1.cache.v, d1.block_table, d1.seqlens,
                                   max_seqlen_k=ctx, scale=di.scale, causal=causal, err=err)
    # fused path on a fresh copy of the same cache
    d2 = di.to("cuda")
    o2, l2 = pkv.paged_decode_attn_append(d2.q, kn.cuda(), vn.cuda(), d2.cache.k, d2.cache.v,
                                          d2.block_table, d2.seqlens, max_seqlen_k=ctx,
                                          scale=di.scale, causal=causal, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for b1, b2 in zip(d1.cache.backing, d2.cache.backing):
        assert bits_equal(b1.cpu(), b2.cpu()), "cache contents differ"
    assert bits_equal(o1.cpu(), o2.cpu()) and bits_equal(l1.cpu(), l2.cpu())
    # and the result is right: oracle append, then oracle attention
    host = di.cache.clone()
    oracle.kv_append(kn, vn, host.k, host.v, di.block_table, di.seqlens - n)
    ref_o, ref_l = oracle.paged_attn(di.q, host.k, host.v, di.block_table, di.seqlens, di.scale,
                                     causal)
    assert_close_to_oracle(o2.cpu(), l2.cpu(), ref_o, ref_l)


def test_fused_append_rejects_bad_counts():
    di = I.p2_case(1, 1, 64, 4, 2, 128, 16, causal=False, seed=5, seqlens=[64]).to("cuda")
    kn = torch.zeros(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_decode_attn_append(di.q, kn, kn, di.cache.k, di.cache.v, di.block_table,
                                     di.seqlens, max_seqlen_k=64)
