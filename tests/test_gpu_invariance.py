"""Bitwise invariances of the CUDA path (through the C ABI).

* batch = 1 vs batch = N, and padding layouts (wider tables with junk past
  the last used block, extra cache blocks, blocks moved elsewhere) -- the
  [WS1] "KV-cache path consistency (prefill & decode)" acceptance list;
* contiguous vs interleaved non-contiguous cache -- ROCm/aiter d293d61 "pin
  non-contiguous paged KV block stride" asserts < 1e-5, here bit for bit;
* decode row t == causal prefill row t, multi-query decode rows == prefill
  rows, chunked prefill == full prefill ("generate then re-score"), with the
  cache filled by kv_append in steps, as in jouleclaw's
  inplace_incremental_decode_matches_one_shot_prefill;
* kv_append stores the bits the oracle's append stores.
"""
import pytest
import torch

import oracle
import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal, oracle_of, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,causal,sq", [(128, False, 1), (64, True, 3), (128, True, 17)])
def test_interleaved_equals_contiguous_bitwise(d, causal, sq):
    di = I.p2_case(2, sq, 1024, 6, 3, d, 16, causal=causal, layout="interleaved", seed=31)
    assert not di.cache.k.is_contiguous()
    out1, lse1 = run_gpu(di)
    di2 = I.DecodeInputs(di.q, di.cache.as_contiguous(), di.block_table, di.seqlens, di.Hq,
                         di.Hkv, di.D, di.scale, di.causal)
    out2, lse2 = run_gpu(di2)
    assert bits_equal(out1, out2) and bits_equal(lse1, lse2)


def test_batch_one_equals_batch_n_bitwise():
    gen = torch.Generator().manual_seed(32)
    B = 8
    seqlens = [1, 77, 4096, 4097, 9000, 130, 12000, 2]
    di = I.p2_case(B, 1, 12000, 16, 4, 128, 16, causal=False, layout="interleaved", seed=32,
                   seqlens=seqlens, poison=True)
    out, lse = run_gpu(di)
    for b in range(B):
        one = I.DecodeInputs(di.q[b:b + 1].clone(), di.cache, di.block_table[b:b + 1].clone(),
                             di.seqlens[b:b + 1].clone(), di.Hq, di.Hkv, di.D, di.scale, False)
        o1, l1 = run_gpu(one)
        assert bits_equal(o1[0], out[b]) and bits_equal(l1[0], lse[b]), f"sequence {b}"
    # max_seqlen_k is only a bound: a looser one changes nothing
    o2, l2 = run_gpu(di, max_seqlen_k=30000)
    assert bits_equal(o2, out) and bits_equal(l2, lse)


def test_padding_layouts_bitwise():
    """Same sequences, different padding: a wider table whose unused columns
    hold junk, a cache with extra blocks, and every block moved elsewhere."""
    di = I.p2_case(3, 2, 2000, 8, 2, 128, 16, causal=True, layout="contiguous", seed=33,
                   seqlens=[2000, 513, 1])
    out, lse = run_gpu(di)
    # wider table, junk (-1) past each sequence's last block
    wide = torch.full((3, di.block_table.shape[1] + 40), -1, dtype=torch.int32)
    for b, n in enumerate(di.seqlens.tolist()):
        k = (n + 15) // 16
        wide[b, :k] = di.block_table[b, :k]
    di_w = I.DecodeInputs(di.q, di.cache, wide, di.seqlens, di.Hq, di.Hkv, di.D, di.scale, True)
    o_w, l_w = run_gpu(di_w)
    assert bits_equal(o_w, out) and bits_equal(l_w, lse)
    # extra blocks in the pool and every block moved to a new id
    nb = di.cache.num_blocks
    perm = torch.randperm(nb + 500, generator=torch.Generator().manual_seed(5))[:nb]
    k2 = torch.full((nb + 500, 16, 2, 128), float("nan"), dtype=torch.bfloat16)
    v2 = torch.full((nb + 500, 16, 2, 128), float("nan"), dtype=torch.bfloat16)
    k2[perm] = di.cache.k
    v2[perm] = di.cache.v
    t2 = perm[di.block_table.long()].to(torch.int32)
    di_m = I.DecodeInputs(di.q, I.PagedCache(k2, v2, (k2, v2), "contiguous"), t2, di.seqlens,
                          di.Hq, di.Hkv, di.D, di.scale, True)
    o_m, l_m = run_gpu(di_m)
    assert bits_equal(o_m, out) and bits_equal(l_m, lse)


def test_decode_and_prefill_entry_points_agree_bitwise():
    di = I.p2_case(2, 5, 5000, 8, 2, 128, 16, causal=True, layout="interleaved", seed=34)
    o1, l1 = run_gpu(di, entry=pkv.paged_decode_attn)
    o2, l2 = run_gpu(di, entry=pkv.paged_prefill_attn)
    assert bits_equal(o1, o2) and bits_equal(l1, l2)


def _append(cache, table, k, v, start):
    B = k.shape[0]
    seq = torch.full((B,), start, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_append(k, v, cache.k, cache.v, table, seq, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def _attn(entry, q, cache, table, n, causal=True):
    B = q.shape[0]
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    out, lse = entry(q, cache.k, cache.v, table, seq, max_seqlen_k=n, causal=causal)
    torch.cuda.synchronize()
    return out, lse


def test_generate_then_rescore_bitwise():
    """Chunked prefill (4 x 512 tokens) == full prefill; 64 kv_append + decode
    steps == rows of the re-scoring prefill; multi-query decode (seqlen_q 3 and
    17) == the same prefill rows.  Hq 16 / Hkv 4, D 128, block_size 16, batch 8."""
    cache, table, q_all, k_all, v_all = I.config_parity_cache(device="cuda")
    B = 8
    # chunked prefill, appending each chunk first
    chunk_out, chunk_lse = [], []
    for c in range(4):
        s, e = 512 * c, 512 * (c + 1)
        _append(cache, table, k_all[:, s:e], v_all[:, s:e], s)
        o, l = _attn(pkv.paged_prefill_attn, q_all[:, s:e], cache, table, e)
        chunk_out.append(o)
        chunk_lse.append(l)
    full_o, full_l = _attn(pkv.paged_prefill_attn, q_all[:, :2048], cache, table, 2048)
    assert bits_equal(torch.cat(chunk_out, 1).cpu(), full_o.cpu())
    assert bits_equal(torch.cat(chunk_lse, 2).cpu(), full_l.cpu())
    # 64 decode steps
    dec_o, dec_l = [], []
    for t in range(2048, 2048 + 64):
        _append(cache, table, k_all[:, t:t + 1], v_all[:, t:t + 1], t)
        o, l = _attn(pkv.paged_decode_attn, q_all[:, t:t + 1], cache, table, t + 1)
        dec_o.append(o)
        dec_l.append(l)
    # 17 more tokens, then the multi-query decodes
    T = 2048 + 64 + 17
    _append(cache, table, k_all[:, 2112:T], v_all[:, 2112:T], 2112)
    mq17_o, mq17_l = _attn(pkv.paged_decode_attn, q_all[:, T - 17:T], cache, table, T)
    mq3_o, mq3_l = _attn(pkv.paged_decode_attn, q_all[:, T - 3:T], cache, table, T)
    # re-score everything with one causal prefill
    re_o, re_l = _attn(pkv.paged_prefill_attn, q_all[:, :T], cache, table, T)
    re_o, re_l = re_o.cpu(), re_l.cpu()
    assert bits_equal(re_o[:, :2048], full_o.cpu()) and bits_equal(re_l[:, :, :2048], full_l.cpu())
    for k, t in enumerate(range(2048, 2112)):
        assert bits_equal(dec_o[k][:, 0].cpu(), re_o[:, t]), f"decode step {t}"
        assert bits_equal(dec_l[k][:, :, 0].cpu(), re_l[:, :, t]), f"decode step {t} lse"
    assert bits_equal(mq17_o.cpu(), re_o[:, T - 17:T]) and bits_equal(mq17_l.cpu(), re_l[:, :, T - 17:T])
    assert bits_equal(mq3_o.cpu(), re_o[:, T - 3:T]) and bits_equal(mq3_l.cpu(), re_l[:, :, T - 3:T])
    # and the re-scored rows are right: oracle on two sequences
    host = I.DecodeInputs(q_all[:2, :T].cpu(), cache.to("cpu"), table[:2].cpu(),
                          torch.full((2,), T, dtype=torch.int32), 16, 4, 128,
                          1.0 / 128 ** 0.5, True)
    ref_o, ref_l = oracle_of(host)
    assert_close_to_oracle(re_o[:2], re_l[:2], ref_o, ref_l)


@pytest.mark.parametrize("layout", ["contiguous", "interleaved"])
@pytest.mark.parametrize("n_new", [1, 7, 512])
def test_kv_append_matches_oracle_bits(layout, n_new):
    gen = torch.Generator().manual_seed(40 + n_new)
    di = I.p2_case(3, 1, 2000, 8, 4, 128, 16, causal=False, layout=layout, seed=41,
                   seqlens=[0, 100, 1400])
    kn = I.randn_bf16((3, n_new, 4, 128), gen)
    vn = I.randn_bf16((3, n_new, 4, 128), gen)
    ref = di.cache.clone()
    oracle.kv_append(kn, vn, ref.k, ref.v, di.block_table, di.seqlens)
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_append(kn.cuda(), vn.cuda(), d.cache.k, d.cache.v, d.block_table, d.seqlens, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert bits_equal(d.cache.k.cpu(), ref.k) and bits_equal(d.cache.v.cpu(), ref.v)


def test_kv_append_out_of_table_sets_error_flag():
    di = I.p2_case(1, 1, 32, 4, 2, 128, 16, causal=False, seed=42, seqlens=[30]).to("cuda")
    narrow = di.block_table[:, :2].contiguous()          # 32 tokens of room
    kn = torch.zeros(1, 5, 2, 128, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_append(kn, kn, di.cache.k, di.cache.v, narrow, di.seqlens, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.binding.DEVERR_TABLE_WIDTH


def test_short_units_stay_in_step_under_repetition():
    """Several units per CTA, many of them one or two tiles long (causal
    512-token chunks: 512 units of 1-16 tiles per call, so the epilogue of
    one unit overlaps the next units' tiles): repeated chunked prefill equals
    the full prefill bit for bit, every wait completes (no timeout bit) and
    every out / lse element is written (NaN-filled first).  A hand-off
    between the softmax and epilogue warpgroups that could run two units
    ahead showed up here as a timeout and unwritten rows."""
    cache, table, q_all, k_all, v_all = I.config_parity_cache(device="cuda")
    B, Hq, n, c = 8, 16, 2048, 512
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    seq = lambda v: torch.full((B,), v, dtype=torch.int32, device="cuda")
    pkv.kv_append(k_all[:, :n], v_all[:, :n], cache.k, cache.v, table, seq(0), err=err)

    def attn(q, ctx):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, q.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
        return pkv.paged_prefill_attn(q, cache.k, cache.v, table, seq(ctx), max_seqlen_k=ctx,
                                      causal=True, out=out, lse=lse, err=err)

    full_o, full_l = attn(q_all[:, :n], n)
    for rep in range(6):
        outs, lses = [], []
        for s in range(0, n, c):
            o, l = attn(q_all[:, s:s + c], s + c)
            outs.append(o)
            lses.append(l)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"repetition {rep}: device error bits {int(err.item())}"
        co, cl = torch.cat(outs, 1), torch.cat(lses, 2)
        assert not torch.isnan(co.float()).any() and not torch.isnan(cl).any()
        assert bits_equal(co.cpu(), full_o.cpu()) and bits_equal(cl.cpu(), full_l.cpu())
