"""Pins for the CPU fp64 oracle (no GPU).

The oracle is trusted only after it is checked against things other than
itself: hand-derived worked examples (tests/golden/), closed forms
(one visible key, equal scores, two keys), invariants (softmax weights sum to
one, layout / table-permutation / causal-future invariance, decode row equals
last prefill row), and, on special cases, a library routine it does not use
(torch's scaled_dot_product_attention in fp64 over a dense context gathered
with torch indexing, the way the aiter test "pin non-contiguous paged KV block
stride" builds its reference).  Each pin is chosen so that a plausible mistake
in the oracle -- a dropped scale, a wrong GQA head mapping, a transposed
operand, top-left instead of bottom-right causal alignment, an off-by-one in
the padding mask, an over-read past seqlens -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import zlib

import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_decode_31_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_cases.json")


# ---------------------------------------------------------------------------
# independent helpers (torch indexing + torch library attention)
# ---------------------------------------------------------------------------

def torch_dense_gather(view, table_row, n):
    """Dense [n, Hkv, D] context of one sequence via torch indexing (fp64)."""
    bs = view.shape[1]
    nblk = (n + bs - 1) // bs
    blocks = view[table_row[:nblk].long()]                   # [nblk, bs, Hkv, D]
    return blocks.reshape(nblk * bs, *view.shape[2:])[:n].double()


def sdpa_reference(di: I.DecodeInputs):
    """torch SDPA (math backend, fp64) with GQA by repeat_interleave and an
    explicit bottom-right causal + padding mask.  Returns (out, lse)."""
    B, sq, Hq, D = di.q.shape
    G = di.Hq // di.Hkv
    out = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    lse = torch.zeros(B, Hq, sq, dtype=torch.float64)
    for b in range(B):
        n = int(di.seqlens[b])
        K = torch_dense_gather(di.cache.k, di.block_table[b], n)   # [n, Hkv, D]
        V = torch_dense_gather(di.cache.v, di.block_table[b], n)
        K = K.repeat_interleave(G, dim=1).permute(1, 0, 2)          # [Hq, n, D]
        V = V.repeat_interleave(G, dim=1).permute(1, 0, 2)
        q = di.q[b].double().permute(1, 0, 2)                       # [Hq, sq, D]
        pos = torch.arange(sq) + (n - sq)
        mask = torch.ones(sq, n, dtype=torch.bool)
        if di.causal:
            mask = torch.arange(n)[None, :] <= pos[:, None]
        o = F.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=di.scale)
        scores = torch.matmul(q, K.transpose(1, 2)) * di.scale
        scores = scores.masked_fill(~mask, float("-inf"))
        out[b] = o.permute(1, 0, 2)
        lse[b] = torch.logsumexp(scores, dim=-1)
    return out, lse


def run_oracle(di: I.DecodeInputs):
    return oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table,
                             di.seqlens, di.scale, di.causal)


# ---------------------------------------------------------------------------
# worked examples (hand-derived, tests/golden/)
# ---------------------------------------------------------------------------

def _golden_inputs(case):
    D, Hkv = case["D"], case["Hkv"]
    bs, nbk = case["block_size"], case["num_blocks"]
    kc = torch.full((nbk, bs, Hkv, D), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((nbk, bs, Hkv, D), float("nan"), dtype=torch.bfloat16)
    table = torch.tensor(case["block_table"], dtype=torch.int32)
    for j, (kk, vv) in enumerate(zip(case["tokens_k"], case["tokens_v"])):
        blk = int(table[0, j // bs])
        kc[blk, j % bs, 0] = torch.tensor(kk, dtype=torch.bfloat16)
        vc[blk, j % bs, 0] = torch.tensor(vv, dtype=torch.bfloat16)
    q = torch.tensor(case["q"], dtype=torch.bfloat16)
    cache = I.PagedCache(kc, vc, (kc, vc), "contiguous")
    return I.DecodeInputs(q, cache, table, torch.tensor(case["seqlens"], dtype=torch.int32),
                          case["Hq"], Hkv, D, case["scale"], case["causal"])


@pytest.mark.parametrize("idx", [0, 1])
def test_hand_worked_examples(idx):
    case = json.load(open(GOLDEN))["cases"][idx]
    di = _golden_inputs(case)
    out, lse = run_oracle(di)
    exp_out = torch.tensor(case["expected_out"], dtype=torch.float64)
    exp_lse = torch.tensor(case["expected_lse"], dtype=torch.float64)
    assert torch.allclose(out, exp_out, rtol=0, atol=1e-12), (out, exp_out)
    assert torch.allclose(lse, exp_lse, rtol=0, atol=1e-12), (lse, exp_lse)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_single_key_returns_its_value_exactly():
    di = I.p2_case(3, 1, 40, 4, 2, 64, 16, causal=False, seed=1, seqlens=[1, 1, 1])
    out, lse = run_oracle(di)
    G = di.Hq // di.Hkv
    for b in range(di.batch):
        blk = int(di.block_table[b, 0])
        for h in range(di.Hq):
            v = di.cache.v[blk, 0, h // G].double()
            k = di.cache.k[blk, 0, h // G].double().numpy()
            assert torch.equal(out[b, 0, h], v)
            s = di.scale * float(np.dot(di.q[b, 0, h].double().numpy(), k))
            assert abs(float(lse[b, h, 0]) - s) <= 1e-12 * max(1.0, abs(s))


def test_equal_scores_return_mean_of_values_and_log_n():
    di = I.p2_case(2, 1, 300, 6, 3, 128, 16, causal=False, seed=2, seqlens=[300, 77])
    di.q.zero_()
    out, lse = run_oracle(di)
    for b in range(2):
        n = int(di.seqlens[b])
        V = torch_dense_gather(di.cache.v, di.block_table[b], n).numpy()   # [n, Hkv, D]
        for h in range(di.Hq):
            mean = V[:, h // 2, :].mean(axis=0)
            np.testing.assert_allclose(out[b, 0, h].numpy(), mean, rtol=0, atol=1e-12)
            assert abs(float(lse[b, h, 0]) - math.log(n)) < 1e-12


def test_identical_keys_return_mean_of_values():
    di = I.p2_case(1, 1, 64, 2, 1, 64, 16, causal=False, seed=3, seqlens=[50])
    row = di.cache.k[int(di.block_table[0, 0]), 0, 0].clone()
    di.cache.k[:] = row
    out, lse = run_oracle(di)
    V = torch_dense_gather(di.cache.v, di.block_table[0], 50).numpy()
    for h in range(2):
        np.testing.assert_allclose(out[0, 0, h].numpy(), V[:, 0, :].mean(axis=0), atol=1e-12)
        s = di.scale * float(np.dot(di.q[0, 0, h].double().numpy(), row.double().numpy()))
        assert abs(float(lse[0, h, 0]) - (s + math.log(50))) < 1e-12


def test_two_keys_logistic_closed_form():
    di = I.p2_case(1, 1, 2, 1, 1, 64, 16, causal=False, seed=4, seqlens=[2])
    out, lse = run_oracle(di)
    blk = int(di.block_table[0, 0])
    q = di.q[0, 0, 0].double().numpy()
    k0, k1 = (di.cache.k[blk, j, 0].double().numpy() for j in (0, 1))
    v0, v1 = (di.cache.v[blk, j, 0].double().numpy() for j in (0, 1))
    s0, s1 = di.scale * q.dot(k0), di.scale * q.dot(k1)
    w1 = 1.0 / (1.0 + math.exp(s0 - s1))                      # logistic weight of key 1
    np.testing.assert_allclose(out[0, 0, 0].numpy(), (1 - w1) * v0 + w1 * v1, atol=1e-12)
    assert abs(float(lse[0, 0, 0]) - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-12


def test_softmax_weights_sum_to_one_via_one_hot_values():
    """With V_j = e_j (one-hot in d), out[d] is exactly the softmax weight of key d:
    the weights must be positive, sum to 1, and have ratios exp(s_i - s_j)."""
    n, D = 40, 64
    di = I.p2_case(1, 1, n, 2, 1, D, 16, causal=False, seed=5, seqlens=[n])
    di.cache.v.zero_()
    for j in range(n):
        di.cache.v[int(di.block_table[0, j // 16]), j % 16, 0, j] = 1.0
    out, lse = run_oracle(di)
    K = torch_dense_gather(di.cache.k, di.block_table[0], n)[:, 0].numpy()
    for h in range(2):
        w = out[0, 0, h, :n].numpy()
        assert np.all(w > 0) and abs(w.sum() - 1.0) < 1e-12
        assert np.all(out[0, 0, h, n:].numpy() == 0.0)
        s = di.scale * K.dot(di.q[0, 0, h].double().numpy())
        np.testing.assert_allclose(np.log(w) - np.log(w[0]), s - s[0], atol=1e-10)
        np.testing.assert_allclose(float(lse[0, h, 0]), s[0] - math.log(w[0]), atol=1e-10)


# ---------------------------------------------------------------------------
# a library routine on the pages' test grid (small sizes)
# ---------------------------------------------------------------------------

GRID = [(mha, causal, bs, sqk, d)
        for mha in ("mha", "gqa") for causal in (False, True) for bs in (16, 256)
        for sqk in ((1, 339), (3, 1024), (17, 156)) for d in (64, 128)]


@pytest.mark.parametrize("mha,causal,bs,sqk,d", GRID)
def test_matches_torch_sdpa_fp64_on_p2_grid(mha, causal, bs, sqk, d):
    sq, sk = sqk
    Hq = 6
    Hkv = 6 if mha == "mha" else 3
    di = I.p2_case(2, sq, sk, Hq, Hkv, d, bs, causal=causal, layout="interleaved",
                   seed=zlib.crc32(repr((mha, causal, bs, sq, d)).encode()) % 1000, poison=True)
    out, lse = run_oracle(di)
    ref_out, ref_lse = sdpa_reference(di)
    finite = torch.isfinite(ref_lse)
    # rows with no visible key: the pages are silent; the oracle returns 0 / -inf
    assert torch.all(lse[~finite] == float("-inf"))
    empty_rows = (~finite).permute(0, 2, 1)                       # [B, sq, Hq]
    assert torch.all(out[empty_rows] == 0)
    assert torch.allclose(out[~empty_rows], ref_out[~empty_rows], rtol=0, atol=1e-10)
    assert torch.allclose(lse[finite], ref_lse[finite], rtol=0, atol=1e-10)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_interleaved_equals_contiguous_bitwise():
    di = I.p2_case(2, 3, 300, 8, 2, 128, 16, causal=True, layout="interleaved", seed=6)
    assert not di.cache.k.is_contiguous()
    assert di.cache.k.stride(0) == 2 * 16 * 2 * 128
    out1, lse1 = run_oracle(di)
    di2 = I.DecodeInputs(di.q, di.cache.as_contiguous(), di.block_table, di.seqlens,
                         di.Hq, di.Hkv, di.D, di.scale, di.causal)
    out2, lse2 = run_oracle(di2)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_block_table_permutation_with_moved_data_is_invariant():
    di = I.p2_case(2, 1, 500, 4, 2, 64, 16, causal=False, layout="contiguous", seed=7)
    out1, lse1 = run_oracle(di)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(di.cache.num_blocks, generator=g)          # new id of old block i
    k2 = torch.empty_like(di.cache.k)
    v2 = torch.empty_like(di.cache.v)
    k2[perm] = di.cache.k
    v2[perm] = di.cache.v
    table2 = perm[di.block_table.long()].to(torch.int32)
    di2 = I.DecodeInputs(di.q, I.PagedCache(k2, v2, (k2, v2), "contiguous"), table2,
                         di.seqlens, di.Hq, di.Hkv, di.D, di.scale, di.causal)
    out2, lse2 = run_oracle(di2)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_gqa_maps_query_head_to_kv_head_by_floor_division():
    di = I.p2_case(1, 1, 32, 4, 2, 64, 16, causal=False, seed=8, seqlens=[32])
    di.cache.v[:, :, 0] = 1.0
    di.cache.v[:, :, 1] = 2.0
    out, _ = run_oracle(di)
    # (h g) grouping: heads 0,1 -> KV head 0, heads 2,3 -> KV head 1
    for h, want in zip(range(4), (1.0, 1.0, 2.0, 2.0)):
        assert torch.all(out[0, 0, h] == want)


def test_scale_multiplies_the_scores():
    di = I.p2_case(1, 1, 100, 2, 1, 64, 16, causal=False, seed=9, seqlens=[100])
    out1, lse1 = run_oracle(di)
    di2 = I.DecodeInputs(di.q * 2, di.cache, di.block_table, di.seqlens, di.Hq, di.Hkv,
                         di.D, di.scale / 2, di.causal)
    out2, lse2 = run_oracle(di2)
    assert torch.allclose(out1, out2, atol=1e-13) and torch.allclose(lse1, lse2, atol=1e-13)


def test_causal_rows_ignore_future_keys_and_see_their_own():
    n, sq = 70, 5
    di = I.p2_case(1, sq, n, 2, 1, 64, 16, causal=True, seed=10, seqlens=[n])
    out1, lse1 = run_oracle(di)
    # perturb key/value at the last position: only the last row may change
    blk = int(di.block_table[0, (n - 1) // 16])
    di.cache.k[blk, (n - 1) % 16] += 1.0
    di.cache.v[blk, (n - 1) % 16] += 1.0
    out2, lse2 = run_oracle(di)
    assert torch.equal(out1[:, : sq - 1], out2[:, : sq - 1])
    assert not torch.equal(out1[:, sq - 1], out2[:, sq - 1])


def test_decode_row_equals_last_prefill_row():
    """One query against N cached keys reduces exactly like the last row of the
    causal prefill over the same context ([WS1] KV-cache path consistency)."""
    n = 200
    di = I.p2_case(2, n, n, 4, 2, 64, 16, causal=True, seed=11, seqlens=[n, n])
    out_p, lse_p = run_oracle(di)
    for t in (0, 17, 199):
        dd = I.DecodeInputs(di.q[:, t:t + 1].contiguous(), di.cache, di.block_table,
                            torch.tensor([t + 1, t + 1], dtype=torch.int32), di.Hq, di.Hkv,
                            di.D, di.scale, True)
        out_d, lse_d = run_oracle(dd)
        assert torch.equal(out_d[:, 0], out_p[:, t])
        assert torch.equal(lse_d[:, :, 0], lse_p[:, :, t])


def test_rows_with_no_visible_key_return_zero_and_minus_inf():
    di = I.p2_case(1, 17, 20, 2, 1, 64, 16, causal=True, seed=12, seqlens=[5])
    out, lse = run_oracle(di)
    # positions 5-17+i < 0 for i < 12
    assert torch.all(out[0, :12] == 0) and torch.all(lse[0, :, :12] == float("-inf"))
    assert torch.all(torch.isfinite(lse[0, :, 12:]))


def test_nan_in_unused_slots_never_reaches_the_output():
    di = I.p2_case(3, 2, 333, 4, 2, 128, 16, causal=True, seed=13, poison=True)
    assert torch.isnan(di.cache.k.float()).any()
    out, lse = run_oracle(di)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


# ---------------------------------------------------------------------------
# kv_append
# ---------------------------------------------------------------------------

def test_kv_append_writes_bits_at_seqlen_positions():
    g = torch.Generator().manual_seed(14)
    di = I.p2_case(3, 1, 100, 4, 2, 64, 16, causal=False, seed=14, layout="interleaved",
                   seqlens=[10, 31, 0])
    before = di.cache.backing[0].clone()
    n_new = 7
    kn = I.randn_bf16((3, n_new, 2, 64), g)
    vn = I.randn_bf16((3, n_new, 2, 64), g)
    oracle.kv_append(kn, vn, di.cache.k, di.cache.v, di.block_table, di.seqlens)
    touched = torch.zeros(before.shape[:3], dtype=torch.bool)          # [nb, 2, bs]
    for b in range(3):
        for t in range(n_new):
            p = int(di.seqlens[b]) + t
            blk = int(di.block_table[b, p // 16])
            assert torch.equal(di.cache.k[blk, p % 16].view(torch.int16), kn[b, t].view(torch.int16))
            assert torch.equal(di.cache.v[blk, p % 16].view(torch.int16), vn[b, t].view(torch.int16))
            touched[blk, :, p % 16] = True
    after = di.cache.backing[0]
    assert torch.equal(after[~touched].view(torch.int16), before[~touched].view(torch.int16))


def test_kv_append_then_attend_equals_prefilled_cache():
    """P5 pattern: filling the cache in steps [3, 1, 1, 1] and attending equals
    attending over the one-shot filled cache."""
    g = torch.Generator().manual_seed(15)
    B, Hq, Hkv, D, bs = 2, 4, 2, 64, 16
    T = 6
    di = I.p2_case(B, 1, 64, Hq, Hkv, D, bs, causal=True, seed=15, seqlens=[T, T])
    k_all = I.randn_bf16((B, T, Hkv, D), g)
    v_all = I.randn_bf16((B, T, Hkv, D), g)
    q_all = I.randn_bf16((B, T, Hq, D), g)
    # one-shot
    oracle.kv_append(k_all, v_all, di.cache.k, di.cache.v, di.block_table,
                     torch.zeros(B, dtype=torch.int32))
    one = I.DecodeInputs(q_all, di.cache, di.block_table, torch.tensor([T, T], dtype=torch.int32),
                         Hq, Hkv, D, di.scale, True)
    out_one, _ = run_oracle(one)
    # incremental, into a fresh cache
    di.cache.k.fill_(float("nan"))
    di.cache.v.fill_(float("nan"))
    done = 0
    for step in (3, 1, 1, 1):
        oracle.kv_append(k_all[:, done:done + step], v_all[:, done:done + step], di.cache.k,
                         di.cache.v, di.block_table, torch.tensor([done, done], dtype=torch.int32))
        done += step
        inc = I.DecodeInputs(q_all[:, done - step:done], di.cache, di.block_table,
                             torch.tensor([done, done], dtype=torch.int32), Hq, Hkv, D,
                             di.scale, True)
        out_inc, _ = run_oracle(inc)
        assert torch.equal(out_inc, out_one[:, done - step:done])


def test_bad_block_id_is_an_error():
    di = I.p2_case(1, 1, 40, 2, 1, 64, 16, causal=False, seed=16, seqlens=[40])
    di.block_table[0, 1] = di.cache.num_blocks + 5
    with pytest.raises(RuntimeError):
        run_oracle(di)


def test_table_narrower_than_the_context_is_an_error():
    # Column j of a table row holds tokens [j * bs, (j + 1) * bs) (aiter d293d61,
    # _generate_interleaved_block_kvcache: randperm reshaped to (batch, nblocks)).
    # A table whose row is narrower than seqlens[b] / bs does not describe the
    # context: the oracle refuses instead of reading the next row or past the
    # end of the tensor.  Here the last sequence's context needs 3 columns, the
    # table (a column slice, so the row stride stays wider) has 2.
    di = I.p2_case(2, 1, 40, 2, 1, 64, 16, causal=False, seed=17, seqlens=[32, 40])
    narrow = I.DecodeInputs(di.q, di.cache, di.block_table[:, :2], di.seqlens, di.Hq,
                            di.Hkv, di.D, di.scale, di.causal)
    with pytest.raises(RuntimeError, match="status 2"):
        run_oracle(narrow)
    # the same table with both contexts inside its two columns is accepted,
    # and equals the wide table's result for that sequence bit for bit
    fits = I.DecodeInputs(di.q, di.cache, di.block_table[:, :2],
                          torch.tensor([32, 20], dtype=torch.int32), di.Hq, di.Hkv, di.D,
                          di.scale, di.causal)
    wide = I.DecodeInputs(di.q, di.cache, di.block_table,
                          torch.tensor([32, 20], dtype=torch.int32), di.Hq, di.Hkv, di.D,
                          di.scale, di.causal)
    o1, l1 = run_oracle(fits)
    o2, l2 = run_oracle(wide)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
