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

from gpu_helpers import assert_close_to_oracle, bits_equal, oracle_of

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
    # and the CP result is the attention itself: the fp64 oracle over the
    # whole context, 1e-2 on out and 1e-3 on lse
    ro, rl = oracle_of(di)
    assert_close_to_oracle(out.cpu(), lse.cpu(), ro, rl)


@pytest.mark.parametrize("B,sq,ctx,Hq,Hkv,D,bs,causal,world", CASES[1:3])
def test_partial_buffer_holds_the_oracle_split_partials(B, sq, ctx, Hq, Hkv, D, bs, causal, world):
    """Each rank's partial buffer, read through the documented layout
    (dist.partials_views: acc [rows][n_local][D], then (m, l) with m in base-2
    units), holds every reached (row, split)'s partial: the split's own
    attention acc / l and log-sum-exp (m + log2 l) ln 2 match the fp64
    oracle's split_partials (1e-3, the lse bound; the partials are fp32)."""
    import math
    import oracle
    di = I.p2_case(B, sq, max(ctx), Hq, Hkv, D, bs, causal=causal, layout="contiguous",
                   seed=sum(ctx) % 997, seqlens=ctx)
    d = di.to("cuda")
    for r in range(world):
        begin, n_local = pdist.cp_split_share(max(ctx), r, world)
        buf = pkv.paged_attn_partials(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, begin,
                                      n_local, scale=di.scale, causal=causal).cpu()
        acc, ml = pdist.partials_views(buf, B, sq, Hq, D, n_local)
        m_ref, l_ref, a_ref = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table,
                                                    di.seqlens, di.scale, causal, begin, n_local)
        rows = B * sq * Hq
        m_ref, l_ref = m_ref.reshape(rows, n_local), l_ref.reshape(rows, n_local)
        a_ref = a_ref.reshape(rows, n_local, D)
        reached = torch.isfinite(m_ref)
        if not reached.any():
            continue
        lse_gpu = (ml[..., 0].double() + torch.log2(ml[..., 1].double())) * math.log(2.0)
        lse_ref = m_ref + torch.log(l_ref)
        assert (lse_gpu[reached] - lse_ref[reached]).abs().max().item() <= 1e-3
        o_gpu = acc.double() / ml[..., 1:2].double()
        o_ref = a_ref / l_ref.unsqueeze(-1)
        assert (o_gpu[reached] - o_ref[reached]).abs().max().item() <= 1e-3


def test_cp_attention_end_to_end_in_a_one_rank_process_group():
    """dist.cp_attention as a rank runs it -- the split share, the NCCL
    all-gather of the partial buffer and the merge -- in a process group of
    one rank: bitwise the single call, and the oracle's attention."""
    import os
    import socket
    import torch.distributed as dist
    di = I.p2_case(2, 3, 20000, 16, 4, 128, 16, causal=True, layout="contiguous", seed=77,
                   seqlens=[20000, 9000])
    d = di.to("cuda")
    ref_o, ref_l = pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                         max_seqlen_k=20000, scale=di.scale, causal=True)
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    pdist.init("nccl", device=torch.device("cuda:0"), timeout_s=60)
    try:
        out, lse = pdist.cp_attention(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, 20000,
                                      scale=di.scale, causal=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert bits_equal(out.cpu(), ref_o.cpu()) and bits_equal(lse.cpu(), ref_l.cpu())
    ro, rl = oracle_of(di)
    assert_close_to_oracle(out.cpu(), lse.cpu(), ro, rl)


def test_partials_reject_a_small_buffer():
    di = I.p2_case(1, 1, 5000, 8, 2, 128, 16, causal=False, seed=3).to("cuda")
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attn_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens, 0, 2,
                                partials=small)
