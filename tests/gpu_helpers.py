"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and
compare it with the CPU fp64 oracle.

Tolerances: bf16 `out` within 1e-2 max-abs of the fp64 oracle, fp32 `lse`
within 1e-3 (the accuracy bar of the library).  Invariances are bitwise.
"""
import torch

import oracle
import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import inputs as I

ATOL_OUT = 1e-2
ATOL_LSE = 1e-3
NEG_INF = float("-inf")


def run_gpu(di: I.DecodeInputs, entry=None, max_seqlen_k=None, check_err=True):
    """Run one attention call on cuda:0 on a device copy of `di`; returns
    (out, lse) on the CPU."""
    entry = entry or pkv.paged_decode_attn
    d = di.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msk = int(di.seqlens.max()) if max_seqlen_k is None else max_seqlen_k
    out, lse = entry(d.q, d.cache.k, d.cache.v, d.block_table, d.seqlens, max_seqlen_k=msk,
                     scale=di.scale, causal=di.causal, err=err)
    torch.cuda.synchronize()
    if check_err:
        assert int(err.item()) == 0, f"device error bits {int(err.item())}"
    return out.cpu(), lse.cpu()


def oracle_of(di: I.DecodeInputs, b_range=None, kvh_range=None):
    return oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                             di.scale, di.causal, b_range=b_range, kvh_range=kvh_range)


def assert_close_to_oracle(out, lse, ref_out, ref_lse, rows_mask=None):
    """out [B, sq, Hq, D] bf16 vs fp64; lse [B, Hq, sq] fp32 vs fp64.  Rows with
    no visible key must be exactly 0 / -inf.  rows_mask [B, sq, Hq] selects the
    rows the oracle computed (others are NaN in ref)."""
    B, sq, Hq, D = out.shape
    if rows_mask is None:
        rows_mask = torch.ones(B, sq, Hq, dtype=torch.bool)
    ref_lse_r = ref_lse.permute(0, 2, 1)            # [B, sq, Hq]
    lse_r = lse.permute(0, 2, 1).double()
    empty = rows_mask & torch.isneginf(ref_lse_r)
    full = rows_mask & torch.isfinite(ref_lse_r)
    assert torch.all(torch.isneginf(lse_r[empty])), "empty rows must have lse = -inf"
    assert torch.all(out[empty].float() == 0), "empty rows must have out = 0"
    if full.any():
        d_out = (out[full].double() - ref_out[full]).abs().max().item()
        d_lse = (lse_r[full] - ref_lse_r[full]).abs().max().item()
        assert d_out <= ATOL_OUT, f"out max-abs error {d_out:.3e} > {ATOL_OUT}"
        assert d_lse <= ATOL_LSE, f"lse max-abs error {d_lse:.3e} > {ATOL_LSE}"
        return d_out, d_lse
    return 0.0, 0.0


def bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bitwise equality (distinguishes -0 from +0 and compares NaN payloads)."""
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)
