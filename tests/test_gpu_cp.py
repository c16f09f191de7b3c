"""Context parallelism on one GPU: W ranks' shares computed one after another
(pkv_paged_attn_partials, no kernel waits for another), their partial buffers
laid side by side as the all-gather leaves them, and pkv_merge_partials: out
and lse must be bitwise those of the single call over the whole context
(RL-Kernel PR #284 "feat(attention): add CP backward drift validation" reports
CP=2 drift against CP=1; here it is zero by construction).  Each rank's cache
holds only the tokens of its splits -- every other block is NaN -- so a rank
that read outside its share would poison the result."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import dist as pdist
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import bits_equal

pytestmark = pytest.mark.gpu


def _rank_cache(di, begin, n_local, bs):
    """A copy of the cache in which only the blocks holding tokens of splits
    [begin, begin + n_local) keep their values; all others are NaN."""
    c = di.cache.clone()
    keep = torch.zeros(c.k.shape[0], dtype=torch.bool)
    lo, hi = begin * 4096, (begin + n_local) * 4096
    for b in range(di.block_table.shape[0]):
        n = int(di.seqlens[b])
        for j in range(lo // bs, min(hi, n) // bs + 1):
            if j * bs < min(hi, n):
                keep[int(di.block_table[b, j])] = True
    for t in c.backing:
        t[~keep] = float("nan")
    return c


CASES = [
    # (batch, seqlen_q, contexts, Hq, Hkv, D, bs, causal, world)
    (2, 1, [20000, 9000], 32, 8, 128, 16, False, 2),
    (2, 1, [20000, 4097], 32, 8, 128, 16, False, 4),     # ranks past the context: empty shares
    (2, 3, [13000, 12290], 16, 4, 64, 32, True, 3),
    (2, 40, [9000, 5000], 16, 4, 128, 16, True, 2),      # 160 rows per KV head: row-major kernel
]


@pytest.mark.parametrize("B,sq,ctx,Hq,Hkv,D,bs,causal,world", CASES)
def test_context_parallel_equals_single_call_bitwise(B, sq, ctx, Hq, Hkv, D, bs, causal, world):
    di = I.p2_case(B, sq, max(ctx), Hq, Hkv, D, bs, causal=causal, layout="contiguous",
                   seed=sum(ctx) % 991, seqlens=ctx)
    d = di.to("cuda")
    ref_o, ref_l = pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                         max_seqlen_k=max(ctx), scale=di.scale, causal=causal)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    blocks = []
    for r in range(world):
        begin, n_local = pdist.cp_split_share(max(ctx), r, world)
        rc = _rank_cache(di, begin, n_local, bs).to("cuda")
        blocks.append(pkv.paged_attn_partials(d.q, rc.k, rc.v, d.block_table, d.seqlens, begin,
                                              n_local, scale=di.scale, causal=causal, err=err))
        torch.cuda.synchronize()
    gathered = torch.cat(blocks)
    out, lse = pkv.merge_partials(gathered, world, n_local, d.seqlens, tuple(d.q.shape),
                                  causal=causal)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert bits_equal(out.cpu(), ref_o.cpu()) and bits_equal(lse.cpu(), ref_l.cpu())


def test_partials_reject_a_small_buffer():
    di = I.p2_case(1, 1, 5000, 8, 2, 128, 16, causal=False, seed=3).to("cuda")
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attn_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens, 0, 2,
                                partials=small)
