"""Bounded pipeline waits on the GPU (pkv_debug_paged_decode_attn).

Every mbarrier wait in the kernels gives up after a time limit (2 s in every
normal call) and the call then ends with PKV_DEVERR_TIMEOUT in the error word
instead of hanging.  Here the limit is cut to zero, so the first wait that is
not satisfied at once runs out: the call must still return, the error bit
must be set, and the next calls on the same context must compute the right
attention.  No GPU fault is provoked: the kernel takes its own abort path
(each CTA waits for its own copies and MMAs in flight, frees its tensor
memory and leaves)."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import binding
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import assert_close_to_oracle, bits_equal, oracle_of

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_ends_the_call_with_the_timeout_bit():
    di = I.p2_case(4, 1, 20000, 32, 8, 128, 16, causal=False, layout="contiguous", seed=61,
                   seqlens=[20000, 20000, 9000, 20000])
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):  # twice: the first abort leaves nothing behind that breaks the next
        err.zero_()
        binding.debug_paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                        wait_limit_ns=0, max_seqlen_k=20000, scale=di.scale,
                                        err=err)
        torch.cuda.synchronize()
        assert int(err.item()) & binding.DEVERR_TIMEOUT
    # the default limit through the same entry point: no error, the right result,
    # bitwise the normal entry point's
    err.zero_()
    out, lse = binding.debug_paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table,
                                               d.seqlens, wait_limit_ns=2_000_000_000,
                                               max_seqlen_k=20000, scale=di.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref_o, ref_l = pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                         max_seqlen_k=20000, scale=di.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert bits_equal(out.cpu(), ref_o.cpu()) and bits_equal(lse.cpu(), ref_l.cpu())
    ro, rl = oracle_of(di)
    assert_close_to_oracle(out.cpu(), lse.cpu(), ro, rl)
