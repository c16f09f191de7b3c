"""GPU parity of the CUDA path against the CPU fp64 oracle, through the C ABI.

Grid: the aiter test "test(triton/decode): pin non-contiguous paged KV block
stride" (mha/gqa x causal x block_size {16, 256} x (seqlen_q, seqlen_k) in
{(1, 339), (3, 1024), (17, 156)} x D {64, 128}, batch 2, Hq 6, Hkv 3 for gqa),
on the interleaved non-contiguous cache with every unused slot NaN, through
both entry points.  Edge cases: one-token contexts, split boundaries, rows with
no visible key, empty sequences, many splits with a ragged tail.
"""
import zlib

import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, oracle_of, run_gpu

pytestmark = pytest.mark.gpu

GRID = [(mha, causal, bs, sqk, d)
        for mha in ("mha", "gqa") for causal in (False, True) for bs in (16, 256)
        for sqk in ((1, 339), (3, 1024), (17, 156)) for d in (64, 128)]


def test_tiny_config_matches_oracle():
    di = I.config_tiny()
    assert not di.cache.k.is_contiguous() and di.cache.k.stride(0) == 2 * 16 * 2 * 64
    out, lse = run_gpu(di)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("entry", ["decode", "prefill"])
@pytest.mark.parametrize("mha,causal,bs,sqk,d", GRID)
def test_p2_grid_matches_oracle(mha, causal, bs, sqk, d, entry):
    sq, sk = sqk
    Hkv = 6 if mha == "mha" else 3
    di = I.p2_case(2, sq, sk, 6, Hkv, d, bs, causal=causal, layout="interleaved",
                   seed=zlib.crc32(repr((mha, causal, bs, sq, d)).encode()) % 1000, poison=True)
    fn = pkv.paged_decode_attn if entry == "decode" else pkv.paged_prefill_attn
    out, lse = run_gpu(di, entry=fn)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("seqlens", [[1, 1], [4096, 4095], [4097, 8192], [8193, 129],
                                     [12345, 3], [0, 5]])
@pytest.mark.parametrize("d", [64, 128])
def test_split_boundaries_and_edge_lengths(seqlens, d):
    di = I.p2_case(2, 1, max(max(seqlens), 1), 8, 2, d, 16, causal=False, layout="contiguous",
                   seed=sum(seqlens) % 997, seqlens=seqlens, poison=True)
    out, lse = run_gpu(di)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("sq,n", [(17, 5), (40, 40), (3, 2), (64, 4097)])
def test_causal_rows_without_keys_and_long_multi_query(sq, n):
    di = I.p2_case(2, sq, n, 4, 1, 128, 16, causal=True, layout="interleaved", seed=sq + n,
                   seqlens=[n, max(n - 1, 1)], poison=True)
    out, lse = run_gpu(di, entry=pkv.paged_prefill_attn)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_query_group_sizes(G):
    Hkv = 2
    di = I.p2_case(3, 1, 700, G * Hkv, Hkv, 128, 32, causal=False, layout="interleaved",
                   seed=G, poison=True)
    out, lse = run_gpu(di)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("bs", [16, 32, 64, 128, 256])
def test_block_sizes(bs):
    di = I.p2_case(2, 2, 1500, 8, 4, 128, bs, causal=True, layout="interleaved", seed=bs,
                   poison=True)
    out, lse = run_gpu(di)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


def test_head_major_cache_layout():
    """A cache laid out [num_blocks, Hkv, block_size, D] (head stride larger
    than slot stride) viewed as [num_blocks, block_size, Hkv, D]."""
    di = I.p2_case(2, 1, 600, 8, 4, 128, 16, causal=False, layout="contiguous", seed=21,
                   poison=True)
    k_hm = di.cache.k.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    v_hm = di.cache.v.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    assert k_hm.stride(2) > k_hm.stride(1)
    di2 = I.DecodeInputs(di.q, I.PagedCache(k_hm, v_hm, (k_hm, v_hm), "contiguous"),
                         di.block_table, di.seqlens, di.Hq, di.Hkv, di.D, di.scale, di.causal)
    out, lse = run_gpu(di2)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


def test_strided_query_and_output():
    """q taken from a fused [B, s, (Hq + 2 Hkv) * D] projection output, out
    written into a wider buffer: only the strides change."""
    di = I.p2_case(2, 3, 300, 8, 2, 128, 16, causal=True, layout="interleaved", seed=22)
    qkv = torch.zeros(2, 3, 12, 128, dtype=torch.bfloat16)
    qkv[:, :, :8] = di.q
    d = di.to("cuda")
    q_view = qkv.cuda()[:, :, :8]
    assert not q_view.is_contiguous()
    out_buf = torch.full((2, 3, 10, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out_view = out_buf[:, :, 1:9]
    lse = torch.empty(2, 8, 3, dtype=torch.float32, device="cuda")
    pkv.paged_decode_attn(q_view, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                          max_seqlen_k=300, scale=di.scale, causal=True, out=out_view, lse=lse)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle_of(di)
    out = out_buf.cpu()
    assert torch.all(out[:, :, 0] == 7.0) and torch.all(out[:, :, 9] == 7.0)
    assert_close_to_oracle(out[:, :, 1:9].contiguous(), lse.cpu(), ref_out, ref_lse)


def test_argument_errors_raise_and_launch_nothing():
    di = I.p2_case(1, 1, 64, 4, 2, 128, 16, causal=False, seed=23).to("cuda")
    with pytest.raises(pkv.PagedKVError):  # workspace too small
        pkv.paged_decode_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                              max_seqlen_k=64, workspace=torch.empty(16, dtype=torch.uint8,
                                                                     device="cuda"))
    with pytest.raises(pkv.PagedKVError):  # Hq % Hkv != 0
        q3 = torch.zeros(1, 1, 3, 128, dtype=torch.bfloat16, device="cuda")
        pkv.paged_decode_attn(q3, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                              max_seqlen_k=64)
    with pytest.raises(pkv.PagedKVError):  # head_dim 96
        kc = torch.zeros(8, 16, 2, 96, dtype=torch.bfloat16, device="cuda")
        q96 = torch.zeros(1, 1, 4, 96, dtype=torch.bfloat16, device="cuda")
        pkv.paged_decode_attn(q96, kc, kc, di.block_table, di.seqlens, max_seqlen_k=64)


def test_bad_block_ids_set_the_error_flag_and_do_not_fault():
    di = I.p2_case(2, 1, 300, 4, 2, 128, 16, causal=False, seed=24, seqlens=[300, 200])
    di.block_table[0, 3] = di.cache.num_blocks + 100
    di.block_table[1, 5] = -7
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, max_seqlen_k=300,
                          err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.binding.DEVERR_BAD_BLOCK
    # the context is still usable
    out, lse = run_gpu(I.config_tiny())
    assert torch.isfinite(out.float()).all()


def test_table_too_narrow_sets_the_error_flag():
    di = I.p2_case(1, 1, 300, 4, 2, 128, 16, causal=False, seed=25, seqlens=[300])
    d = di.to("cuda")
    narrow = d.block_table[:, :10].contiguous()        # covers 160 tokens only
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, narrow, d.seqlens, max_seqlen_k=300,
                          err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.binding.DEVERR_TABLE_WIDTH


@pytest.mark.parametrize("entry", ["decode", "prefill"])
def test_short_contexts_stay_in_bounds_over_seeds(entry):
    """Short causal contexts where one or two keys carry most of the weight:
    the case where bf16 rounding of P alone (without its low part) pushed
    out past the 1e-2 bound.  24 seeds of the (gqa, causal, block_size 256,
    seqlen_q 17, contexts <= 156, D 128) grid case."""
    fn = pkv.paged_decode_attn if entry == "decode" else pkv.paged_prefill_attn
    worst = 0.0
    for seed in range(24):
        di = I.p2_case(2, 17, 156, 6, 3, 128, 256, causal=True, layout="interleaved",
                       seed=500 + seed, poison=True)
        out, lse = run_gpu(di, entry=fn)
        ref_out, ref_lse = oracle_of(di)
        d_out, _ = assert_close_to_oracle(out, lse, ref_out, ref_lse)
        worst = max(worst, d_out)
    assert worst <= 1e-2


@pytest.mark.parametrize("sq", [1, 64])          # transposed kernel / row-major kernel
def test_context_longer_than_max_seqlen_k_sets_the_error_flag(sq):
    """max_seqlen_k sizes the split grid on the host; a sequence longer than
    it is a caller error the device reports (PKV_DEVERR_SEQ_LEN) instead of
    returning a silently truncated attention.  A bound that covers every
    context leaves the error word at zero."""
    di = I.p2_case(2, sq, 9000, 16, 4, 128, 16, causal=True, layout="contiguous", seed=26,
                   seqlens=[9000, 3000])
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for fn in (pkv.paged_decode_attn, pkv.paged_prefill_attn):
        err.zero_()
        fn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, max_seqlen_k=5000,
           scale=di.scale, causal=True, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == pkv.binding.DEVERR_SEQ_LEN
        err.zero_()
        out, lse = fn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, max_seqlen_k=9000,
                      scale=di.scale, causal=True, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    # the backward sizes its key tiles from the same bound and flags the same way
    dout = torch.randn(out.shape, dtype=torch.bfloat16, device="cuda")
    err.zero_()
    pkv.paged_prefill_attn_bwd(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, out, lse, dout,
                               max_seqlen_k=5000, scale=di.scale, causal=True, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pkv.binding.DEVERR_SEQ_LEN


def _growing_keys(di, growth):
    """Scale every cached key at position pos by 1 + growth * (pos // 128), so
    that each 128-token tile's scores are larger than the last tile's."""
    k = di.cache.k
    bs = di.cache.block_size
    for b, n in enumerate(di.seqlens.tolist()):
        pos = torch.arange(n)
        blk = di.block_table[b, pos // bs].long()
        f = (1.0 + growth * (pos // 128).float()).to(torch.bfloat16)
        k[blk, pos % bs] = (k[blk, pos % bs].float() * f[:, None, None].float()).to(torch.bfloat16)


def _max_rises(di):
    """How often, over every (sequence, query row, query head), a tile's max
    score (base 2) exceeds the split's running max by more than 8 after the
    split's first tile -- the case where the accumulators are rescaled in
    place (the running max follows the kernels' rule: it rises to a tile's
    max only past that slack)."""
    import math
    G = di.Hq // di.Hkv
    rises = 0
    for b, n in enumerate(di.seqlens.tolist()):
        pos = torch.arange(n)
        blk = di.block_table[b, pos // di.cache.block_size].long()
        kk = di.cache.k[blk, pos % di.cache.block_size].double()        # [n, Hkv, D]
        q = di.q[b].double()                                             # [sq, Hq, D]
        s = torch.einsum("qhd,nhd->qhn", q, kk.repeat_interleave(G, dim=1)) * di.scale / math.log(2)
        sq = q.shape[0]
        for i in range(sq):
            lim = n - sq + i + 1 if di.causal else n
            m = torch.full((di.Hq,), float("-inf"), dtype=torch.float64)
            for t0 in range(0, lim, 128):
                if t0 % 4096 == 0:
                    m.fill_(float("-inf"))
                tm = s[i, :, t0:min(lim, t0 + 128)].max(dim=1).values
                rises += int(((m > float("-inf")) & (tm > m + 8)).sum())
                m = torch.where(tm > m + 8, tm, m)
    return rises


@pytest.mark.parametrize("sq,causal,n,d", [(1, False, 2200, 128), (3, True, 2200, 128),
                                            (16, True, 2200, 128), (150, True, 2200, 128),
                                            (1, False, 9000, 128), (150, True, 9000, 128),
                                            (3, True, 2200, 64), (150, True, 2200, 64)])
def test_rising_maxima_rescale_in_place_and_match_oracle(sq, causal, n, d):
    """Keys that grow tile by tile: a row's max rises past the 2^8 slack at
    almost every tile, so the accumulators are rescaled in TMEM between tiles
    (transposed kernel at seqlen_q 1, 3 and 16 -- 64 rows per KV head --,
    row-major kernel at 150 x G 4 rows; head_dim 64 and 128; 9000-token
    contexts: three splits, the running max restarting at each, and the
    merge).  Against the oracle; the decode row equals the causal
    prefill's last row.  The softmax here is nearly one-hot, so out is close
    to a single V row and can exceed 4 in magnitude, where bf16's own rounding
    of the exact result reaches 2^-6 = 1.6e-2: out is held to 1e-2 plus half
    a bf16 unit in the last place of the oracle's value (2^-8 |ref|)."""
    di = I.p2_case(2, sq, n, 16, 4, d, 16, causal=causal, layout="interleaved", seed=71,
                   seqlens=[n, (n * 3) // 5])
    _growing_keys(di, 2.5)
    assert _max_rises(di) > 0
    out, lse = run_gpu(di, entry=pkv.paged_prefill_attn)
    ref_out, ref_lse = oracle_of(di)
    assert torch.isfinite(ref_lse).all() and torch.isfinite(lse).all()
    err = (out.double() - ref_out).abs()
    assert (err <= 1e-2 + ref_out.abs() * 2.0 ** -8).all(), f"out max-abs error {err.max():.3e}"
    assert (lse.double() - ref_lse).abs().max() <= 1e-3
    if causal:
        last = I.DecodeInputs(di.q[:, -1:].contiguous(), di.cache, di.block_table, di.seqlens,
                              di.Hq, di.Hkv, di.D, di.scale, True)
        o1, l1 = run_gpu(last, entry=pkv.paged_decode_attn)
        from gpu_helpers import bits_equal
        assert bits_equal(o1, out[:, -1:].contiguous()) and bits_equal(l1, lse[:, :, -1:].contiguous())
