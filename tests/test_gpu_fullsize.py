"""Parity at the workloads' full sizes, in the launch configuration the bench
uses (the same entry points, persistent grid, workspace), on sampled rows the
oracle computes one (sequence, KV head) at a time: the GQA decode shard, the
ragged batch (block_size 256, interleaved, NaN tails and spare blocks) and the
long-context batch through the fused append + decode call the bench times."""
import pytest
import torch

import oracle
import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal, run_gpu

pytestmark = pytest.mark.gpu


def _sampled_check(di_host, out, lse, seqs, kv_heads):
    G = di_host.Hq // di_host.Hkv
    for b in seqs:
        for h0, h1 in kv_heads:
            ref_o, ref_l = oracle.paged_attn(di_host.q, di_host.cache.k, di_host.cache.v,
                                             di_host.block_table, di_host.seqlens, di_host.scale,
                                             di_host.causal, b_range=(b, b + 1), kvh_range=(h0, h1))
            mask = torch.zeros(out.shape[:3], dtype=torch.bool)
            mask[b, :, h0 * G:h1 * G] = True
            assert_close_to_oracle(out, lse, ref_o, ref_l, rows_mask=mask)


def test_gqa_shard_full_size():
    di = I.config_gqa_shard()
    out, lse = run_gpu(di)
    _sampled_check(di, out, lse, seqs=[0, 17, 31], kv_heads=[(0, 2), (6, 8)])


def test_ragged_full_size():
    di = I.config_ragged()
    assert torch.isnan(di.cache.k.float()).any()
    out, lse = run_gpu(di, max_seqlen_k=32768)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    sl = di.seqlens.tolist()
    picks = sorted({sl.index(min(sl)), sl.index(max(sl)), 5, 40})
    _sampled_check(di, out, lse, seqs=picks, kv_heads=[(0, 4)])


def test_long_context_full_size_fused_append():
    """Exactly the bench's step: seed 1000, 131072-token contexts, the newest
    token appended inside the decode call."""
    dev = torch.device("cuda", 0)
    di = I.config_long_context(seed=1000, device=dev)
    gen = torch.Generator(device=dev).manual_seed(2000)
    kn = torch.randn(4, 1, 8, 128, generator=gen, device=dev).to(torch.bfloat16)
    vn = torch.randn(4, 1, 8, 128, generator=gen, device=dev).to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = pkv.paged_decode_attn_append(di.q, kn, vn, di.cache.k, di.cache.v, di.block_table,
                                            di.seqlens, max_seqlen_k=131072, scale=di.scale,
                                            causal=False, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    host = I.DecodeInputs(di.q.cpu(), di.cache.to("cpu"), di.block_table.cpu(), di.seqlens.cpu(),
                          32, 8, 128, di.scale, False)
    del di
    torch.cuda.empty_cache()
    # the appended token is in the host copy of the cache (copied after the call)
    _sampled_check(host, out.cpu(), lse.cpu(), seqs=[0, 3], kv_heads=[(0, 1), (7, 8)])


def test_million_token_contexts():
    """The longest contexts tested: 2^20 tokens (256 splits per row) and
    2^20 - 4097 (a last split of 4095 keys), Hq 8 / Hkv 2, D 128, block size
    16, contiguous cache with a randperm table.  Every (sequence, KV head)
    group against the oracle; each sequence run alone bitwise equal to its
    rows of the batch (the 256-split merge does not depend on the batch)."""
    dev = torch.device("cuda", 0)
    Hq, Hkv, D, bs, L = 8, 2, 128, 16, 1 << 20
    gen = torch.Generator(device=dev).manual_seed(4242)
    num_blocks = 2 * (L // bs)
    q = I.randn_bf16((2, 1, Hq, D), gen, dev)
    cache = I.make_cache(num_blocks, bs, Hkv, D, "contiguous", gen, dev)
    table = I.randperm_table(num_blocks, 2, gen, dev)
    sl = torch.tensor([L, L - 4097], dtype=torch.int32, device=dev)
    scale = 1.0 / D ** 0.5
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = pkv.paged_decode_attn(q, cache.k, cache.v, table, sl, max_seqlen_k=L, scale=scale,
                                     causal=False, err=err)
    for b in range(2):
        o1, l1 = pkv.paged_decode_attn(q[b:b + 1], cache.k, cache.v, table[b:b + 1], sl[b:b + 1],
                                       max_seqlen_k=L, scale=scale, causal=False, err=err)
        assert bits_equal(o1, out[b:b + 1]) and bits_equal(l1, lse[b:b + 1])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    host = I.DecodeInputs(q.cpu(), cache.to("cpu"), table.cpu(), sl.cpu(), Hq, Hkv, D, scale, False)
    del cache
    torch.cuda.empty_cache()
    _sampled_check(host, out.cpu(), lse.cpu(), seqs=[0, 1], kv_heads=[(0, 1), (1, 2)])
