"""Where the backward's 1e-2 x max|gradient| bound comes from (CPU only).

The GPU backward (pkv_paged_prefill_attn_bwd) computes, per (row, key):
S = q.k in fp32 from bf16 operands, p = 2^(S * c - lse2) in fp32 (c = scale *
log2 e, lse2 = the forward's fp32 lse * log2 e), dP = dout.v in fp32, D = dout
. out in fp32 over the forward's bf16 out, dS = p (dP - D) in fp32; then p and
dS enter the tensor cores as bf16 (dV += P^T dO, dK += dS^T Q, dQ += dS K with
fp32 accumulation), and dq / dk / dv are written as bf16 (dk and dq after one
fp32 multiply by scale).  This file replays exactly those roundings in torch
on the CPU for the cases tests/test_gpu_bwd.py runs and compares them with the
fp64 gradients of oracle.paged_attn_bwd: the replay's error is what the
arithmetic itself costs, and the GPU bound must leave room above it.  The
replay's own sums run in fp64 (the tensor cores' fp32 accumulation adds
errors of order 2^-24 relative, far below the bf16 operand roundings)."""
import math

import pytest
import torch

import oracle
from paged_kv_decode_31_b200 import inputs as I

GPU_BOUND = 1e-2   # tests/test_gpu_bwd.py: max-abs error <= 1e-2 * max|gradient| per tensor

CASES = [
    # the GPU test's cases: (batch, seqlen_q, contexts, Hq, Hkv, D, bs, causal, layout)
    (2, 40, [300, 160], 16, 4, 128, 16, True, "interleaved"),
    (2, 130, [700, 130], 8, 2, 64, 32, True, "contiguous"),
    (1, 64, [5000], 8, 8, 128, 64, False, "contiguous"),
    (3, 17, [33, 17, 900], 32, 8, 128, 16, True, "interleaved"),
]


def _bf16(x):
    return x.to(torch.bfloat16).to(torch.float64)


def _f32(x):
    return x.to(torch.float32).to(torch.float64)


def replay_bwd(di, dout, causal):
    """The GPU backward's roundings, replayed: returns (dq, dk, dv) like
    oracle.paged_attn_bwd (dk / dv by token position)."""
    out, lse = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                 di.scale, causal)
    out_b = _bf16(out)                        # the forward writes out as bf16 ...
    lse_f = _f32(lse)                         # ... and lse as fp32
    B, sq, Hq, D = di.q.shape
    Hkv, G, bs = di.Hkv, di.Hq // di.Hkv, di.cache.block_size
    c = float(torch.tensor(di.scale * 1.4426950408889634, dtype=torch.float32))
    scale = float(torch.tensor(di.scale, dtype=torch.float32))
    Lmax = int(di.seqlens.max())
    dq = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    dk = torch.zeros(B, Lmax, Hkv, D, dtype=torch.float64)
    dv = torch.zeros(B, Lmax, Hkv, D, dtype=torch.float64)
    for b in range(B):
        n = int(di.seqlens[b])
        j = torch.arange(n)
        blk = di.block_table[b, j // bs].long()
        K = di.cache.k[blk, j % bs].double()
        V = di.cache.v[blk, j % bs].double()
        pos = n - sq + torch.arange(sq)
        vis = torch.ones(sq, n, dtype=torch.bool)
        if causal:
            vis = j[None, :] <= pos[:, None]
        for g in range(Hkv):
            acc_k = torch.zeros(n, D, dtype=torch.float64)
            acc_v = torch.zeros(n, D, dtype=torch.float64)
            for h in range(g * G, (g + 1) * G):
                Q = di.q[b, :, h].double()
                dO = dout[b, :, h].double()
                S = _f32(Q @ K[:, g].T)
                lse2 = _f32(lse_f[b, h] * 1.4426950408889634)
                P = _f32(torch.exp2(_f32(_f32(S * c) - lse2[:, None])))
                P = torch.where(vis, P, torch.zeros_like(P))
                dP = _f32(dO @ V[:, g].T)
                Dd = _f32((dO * out_b[b, :, h]).sum(dim=1))
                dS = _f32(P * _f32(dP - Dd[:, None]))
                Pb, dSb = _bf16(P), _bf16(dS)
                acc_v += Pb.T @ dO
                acc_k += dSb.T @ Q
                dq[b, :, h] = _bf16(_f32(_f32(dSb @ K[:, g]) * scale))
            dk[b, :n, g] = _bf16(_f32(_f32(acc_k) * scale))
            dv[b, :n, g] = _bf16(_f32(acc_v))
    return dq, dk, dv


@pytest.mark.parametrize("trial", [0, 1, 2])
@pytest.mark.parametrize("B,sq,ctx,Hq,Hkv,D,bs,causal,layout", CASES)
def test_replayed_roundings_stay_well_inside_the_gpu_bound(B, sq, ctx, Hq, Hkv, D, bs, causal,
                                                           layout, trial):
    # trial 0 is the GPU test's own input (its seeds); 1 and 2 are fresh draws
    di = I.p2_case(B, sq, max(ctx), Hq, Hkv, D, bs, causal=causal, layout=layout,
                   seed=sum(ctx) + sq + 1000 * trial, seqlens=ctx)
    dout = I.randn_bf16((B, sq, Hq, D), torch.Generator().manual_seed(sq + D + 1000 * trial))
    ref = oracle.paged_attn_bwd(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                di.scale, causal, dout)
    got = replay_bwd(di, dout, causal)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        L = min(g.shape[1], r.shape[1])
        rel = float((g[:, :L] - r[:, :L]).abs().max()) / max(float(r.abs().max()), 1e-3)
        # the bf16 roundings cost 2e-3 .. 5.5e-3 of max|gradient| on these
        # cases; the GPU bound stays above what the arithmetic itself costs
        # by a factor of at least 1/0.6
        assert rel <= 0.6 * GPU_BOUND, f"{name}: replayed error {rel:.2e} of max|gradient|"
        # and the replay really does round (a replay that matched the oracle
        # exactly would say nothing about the bound)
        assert rel > 1e-4, f"{name}: replay shows no rounding at all ({rel:.1e})"
