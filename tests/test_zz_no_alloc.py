"""The allocation-free decode entry point (pkv_paged_decode_attn_static_ws).

It serves callers that cannot allocate device memory when they call; its
scratch is a device array owned by the library and shared by every call.  This
file is collected last on purpose, so that a run stopping at the first failure
has already run every other test; it passes on its own in a fresh process too.
"""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import binding
from paged_kv_decode_31_b200 import inputs as I

from gpu_helpers import ATOL_LSE, ATOL_OUT, bits_equal

pytestmark = pytest.mark.gpu


def _reference(d, msk):
    return pkv.paged_decode_attn(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                 max_seqlen_k=msk, scale=d.scale, causal=d.causal)


def _static(d, msk):
    out = torch.empty_like(d.q)
    lse = torch.empty(d.batch, d.Hq, d.seqlen_q, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.paged_decode_attn_static_ws(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens,
                                        max_seqlen_k=msk, scale=d.scale, causal=d.causal,
                                        out=out, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out, lse


def test_static_workspace_matches_workspace_entry_two_calls_in_a_row():
    # two different problems back to back: the second call finds the first
    # call's partials in the shared scratch and must not be affected by them
    cases = [I.p2_case(4, 1, 20000, 32, 8, 128, 16, causal=False, layout="contiguous", seed=91,
                       poison=True),
             I.p2_case(2, 3, 9000, 16, 4, 64, 256, causal=True, layout="interleaved", seed=92,
                       poison=True)]
    for di in cases:
        d = di.to("cuda")
        msk = int(di.seqlens.max())
        ref_out, ref_lse = _reference(d, msk)
        out, lse = _static(d, msk)
        torch.cuda.synchronize()
        assert (out.float() - ref_out.float()).abs().max().item() <= ATOL_OUT
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (lse[fin] - ref_lse[fin]).abs().max().item() <= ATOL_LSE
        assert bits_equal(out.cpu(), ref_out.cpu()) and bits_equal(lse.cpu(), ref_lse.cpu())


def test_static_workspace_rejects_problems_beyond_its_size():
    di = I.p2_case(1, 1, 64, 4, 2, 128, 16, causal=False, seed=93).to("cuda")
    # batch 64 x seqlen_q 64 x Hq 32 rows x 4 splits of 130 floats > 8 MiB
    q = torch.zeros(64, 64, 32, 128, dtype=torch.bfloat16, device="cuda")
    assert pkv.workspace_size(64, 64, 32, 128, 16384) > binding.STATIC_WORKSPACE_BYTES
    with pytest.raises(pkv.PagedKVError):
        binding.paged_decode_attn_static_ws(
            q, di.cache.k, di.cache.v, di.block_table.expand(64, -1).contiguous(),
            di.seqlens.expand(64).contiguous(), max_seqlen_k=16384, out=torch.empty_like(q),
            lse=torch.empty(64, 32, 64, dtype=torch.float32, device="cuda"))
    # the C entry point itself returns PKV_ERR_WORKSPACE and launches nothing;
    # every pointer is a real device buffer of the sizes passed, so even a call
    # that got past the size check could only touch memory it owns
    import ctypes
    fn = binding.lib().pkv_paged_decode_attn_static_ws
    assert fn.argtypes  # set by the binding call above
    table = di.block_table.expand(64, -1).contiguous()
    seqlens = di.seqlens.expand(64).contiguous()
    out = torch.empty_like(q)
    lse = torch.empty(64, 32, 64, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = (ctypes.c_int64 * 3)(*q.stride()[:3])
    kst = (ctypes.c_int64 * 3)(*di.cache.k.stride()[:3])
    vst = (ctypes.c_int64 * 3)(*di.cache.v.stride()[:3])
    ost = (ctypes.c_int64 * 3)(*out.stride()[:3])
    rc = fn(q.data_ptr(), st, di.cache.k.data_ptr(), kst, di.cache.v.data_ptr(), vst,
            di.cache.k.shape[0], table.data_ptr(), table.stride(0), table.shape[1],
            seqlens.data_ptr(), 16384, 64, 64, 32, 2, 128, 16, 0.088, 0, out.data_ptr(), ost,
            lse.data_ptr(), err.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 2  # PKV_ERR_WORKSPACE
    assert int(err.item()) == 0
