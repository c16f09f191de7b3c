"""The row-major split kernel, which serves calls with more than 64 rows (query
heads x query tokens) per KV head when the query group G divides 128: parity
with the oracle on its direct-write path (one split) and its merge path (several
splits), rows with no visible key, G = 1 / 16 / 32, strided and head-major q,
an unaligned strided out; and bit-equality of its rows with the transposed
kernel that serves 64 rows or fewer (the same rows of the same call shape, cut
down to the last query tokens)."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal, oracle_of, run_gpu

pytestmark = pytest.mark.gpu


def _last_tokens(di, n):
    return I.DecodeInputs(di.q[:, -n:].contiguous(), di.cache, di.block_table, di.seqlens,
                          di.Hq, di.Hkv, di.D, di.scale, di.causal)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("ctx", [3000, 9000])   # one split (direct write) / three (merge)
def test_rows_kernel_matches_oracle(d, ctx):
    di = I.p2_case(3, 40, ctx, 16, 4, d, 16, causal=True, layout="interleaved", seed=ctx + d,
                   seqlens=[ctx, ctx - 1000, 30], poison=True)  # 30 < 40: rows with no key
    out, lse = run_gpu(di, entry=pkv.paged_prefill_attn)
    ref_out, ref_lse = oracle_of(di)
    assert torch.isneginf(ref_lse[2, :, :10]).all()
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("ctx", [3000, 9000])
@pytest.mark.parametrize("causal", [True, False])
def test_rows_kernel_equals_transposed_kernel_bitwise(ctx, causal):
    di = I.p2_case(2, 40, ctx, 16, 4, 128, 16, causal=causal, layout="contiguous",
                   seed=ctx + 7, seqlens=[ctx, ctx - 77])
    o_big, l_big = run_gpu(di)              # 160 rows per KV head: row-major kernel
    for n in (16, 4):                       # 64 rows (N = 64) and 16 rows (N = 16)
        o, l = run_gpu(_last_tokens(di, n))
        assert bits_equal(o, o_big[:, -n:]), f"out of the last {n} tokens"
        assert bits_equal(l, l_big[:, :, -n:]), f"lse of the last {n} tokens"


@pytest.mark.parametrize("Hq,Hkv,sq", [(4, 4, 130), (32, 2, 10), (64, 2, 5), (6, 2, 40),
                                       (4, 4, 100), (16, 4, 17)])
def test_rows_kernel_group_sizes(Hq, Hkv, sq):
    """G = 1, 16, 32 in the row-major kernel; G = 3, which does not divide 128,
    and 128 / G query tokens more than seqlen_q (G = 1 with 100 tokens, G = 4
    with 17) in the transposed kernel."""
    di = I.p2_case(2, sq, 1500, Hq, Hkv, 128, 32, causal=True, layout="interleaved",
                   seed=Hq * 100 + sq, poison=True)
    out, lse = run_gpu(di, entry=pkv.paged_prefill_attn)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)


def test_rows_kernel_strided_and_head_major_q():
    di = I.p2_case(2, 48, 2500, 8, 2, 128, 16, causal=True, layout="interleaved", seed=61)
    ref_out, ref_lse = oracle_of(di)
    d = di.to("cuda")
    # q from a fused [B, s, (Hq + 2 Hkv), D] projection
    qkv = torch.zeros(2, 48, 12, 128, dtype=torch.bfloat16, device="cuda")
    qkv[:, :, :8] = d.q
    out, lse = pkv.paged_prefill_attn(qkv[:, :, :8], d.cache.k, d.cache.v, d.block_table,
                                      d.seqlens, max_seqlen_k=2500, scale=di.scale, causal=True)
    torch.cuda.synchronize()
    assert_close_to_oracle(out.cpu(), lse.cpu(), ref_out, ref_lse)
    # q stored head-major [B, Hq, s, D] and viewed as [B, s, Hq, D]
    q_hm = d.q.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    assert q_hm.stride(2) > q_hm.stride(1)
    out2, lse2 = pkv.paged_prefill_attn(q_hm, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                        max_seqlen_k=2500, scale=di.scale, causal=True)
    torch.cuda.synchronize()
    assert bits_equal(out2.cpu(), out.cpu()) and bits_equal(lse2.cpu(), lse.cpu())


def test_rows_kernel_unaligned_strided_out():
    """out rows 132 elements apart, starting 8 bytes into the buffer: the
    direct write falls back to element stores."""
    di = I.p2_case(2, 40, 1000, 8, 2, 128, 16, causal=True, layout="contiguous", seed=62)
    d = di.to("cuda")
    buf = torch.full((2, 40, 8, 132), 5.0, dtype=torch.bfloat16, device="cuda")
    out_view = buf[:, :, :, 4:]
    lse = torch.empty(2, 8, 40, dtype=torch.float32, device="cuda")
    pkv.paged_prefill_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                           max_seqlen_k=1000, scale=di.scale, causal=True, out=out_view, lse=lse)
    torch.cuda.synchronize()
    full = buf.cpu()
    assert torch.all(full[..., :4] == 5.0)
    ref_out, ref_lse = oracle_of(di)
    assert_close_to_oracle(full[..., 4:].contiguous(), lse.cpu(), ref_out, ref_lse)
    o_ref, l_ref = run_gpu(di, entry=pkv.paged_prefill_attn)
    assert bits_equal(full[..., 4:].contiguous(), o_ref) and bits_equal(lse.cpu(), l_ref)


def test_rows_kernel_empty_sequences_direct_write():
    """A sequence of length 0 and one shorter than the query chunk, one split:
    every row of the empty sequence is written 0 / -inf by the split kernel."""
    di = I.p2_case(3, 33, 800, 16, 4, 64, 16, causal=True, layout="interleaved", seed=63,
                   seqlens=[800, 0, 20], poison=True)
    out, lse = run_gpu(di, entry=pkv.paged_prefill_attn)
    ref_out, ref_lse = oracle_of(di)
    assert torch.isneginf(lse[1]).all() and torch.all(out[1].float() == 0)
    assert_close_to_oracle(out, lse, ref_out, ref_lse)
