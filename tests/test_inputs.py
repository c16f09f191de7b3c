"""The seeded input recipes (paged_kv_decode_31_b200/inputs.py), checked on
the CPU at reduced sizes: shapes, the randperm block table, the length
distributions, the interleaved layout as two views of one buffer, and NaN
poisoning of exactly the slots no sequence uses.  The same module feeds the
oracle and the CUDA path, so a recipe that drifted would change both sides at
once -- these checks pin it to its stated definition instead."""
import math

import pytest
import torch

from paged_kv_decode_31_b200 import inputs as I


def _used_slots(cache, table, seqlens):
    bs = cache.block_size
    used = torch.zeros(cache.num_blocks, bs, dtype=torch.bool)
    for b, n in enumerate(seqlens.tolist()):
        for j in range(n):
            used[int(table[b, j // bs]), j % bs] = True
    return used


@pytest.mark.parametrize("layout", ["interleaved", "contiguous"])
def test_grid_case_shapes_and_randperm_table(layout):
    di = I.p2_case(3, 2, 1000, 8, 2, 64, 16, causal=True, layout=layout, seed=4)
    nb = math.ceil(1000 / 16) * 3 * 3
    assert tuple(di.q.shape) == (3, 2, 8, 64) and di.q.dtype == torch.bfloat16
    assert tuple(di.cache.k.shape) == (nb, 16, 2, 64) == tuple(di.cache.v.shape)
    assert tuple(di.block_table.shape) == (3, nb // 3) and di.block_table.dtype == torch.int32
    # every block id exactly once: a permutation of range(num_blocks)
    assert torch.equal(di.block_table.flatten().sort().values, torch.arange(nb, dtype=torch.int32))
    assert di.seqlens.dtype == torch.int32 and bool(((di.seqlens >= 1) & (di.seqlens <= 1000)).all())
    assert di.scale == pytest.approx(1 / 8)
    if layout == "interleaved":
        kv = di.cache.backing[0]
        assert tuple(kv.shape) == (nb, 2, 16, 2, 64)
        assert di.cache.k.data_ptr() == kv.data_ptr()
        assert di.cache.v.data_ptr() == kv[:, 1].data_ptr()
        assert di.cache.k.stride(0) == 2 * 16 * 2 * 64  # K and V of a block sit side by side
    else:
        assert di.cache.k.is_contiguous() and di.cache.v.is_contiguous()


def test_same_seed_same_inputs_other_seed_other_inputs():
    a = I.p2_case(2, 1, 300, 4, 2, 64, 16, causal=False, seed=9)
    b = I.p2_case(2, 1, 300, 4, 2, 64, 16, causal=False, seed=9)
    c = I.p2_case(2, 1, 300, 4, 2, 64, 16, causal=False, seed=10)
    assert torch.equal(a.q, b.q) and torch.equal(a.cache.backing[0], b.cache.backing[0])
    assert torch.equal(a.block_table, b.block_table) and torch.equal(a.seqlens, b.seqlens)
    assert not torch.equal(a.q, c.q)


def test_values_are_standard_normal_in_bf16():
    di = I.p2_case(4, 4, 4096, 8, 2, 128, 16, causal=False, layout="contiguous", seed=1)
    x = di.cache.k.float().flatten()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01
    assert torch.equal(x, x.bfloat16().float())


def test_poison_marks_exactly_the_unused_slots():
    di = I.p2_case(3, 1, 100, 4, 2, 64, 16, causal=False, seed=6, seqlens=[100, 33, 1],
                   poison=True)
    used = _used_slots(di.cache, di.block_table, di.seqlens)
    nan = torch.isnan(di.cache.k.float()).all(-1).all(-1)  # [num_blocks, bs]
    assert torch.equal(nan, ~used)
    assert torch.equal(torch.isnan(di.cache.v.float()).all(-1).all(-1), ~used)
    assert not torch.isnan(di.cache.k.float()[used]).any()


def test_tiny_workload_recipe():
    di = I.config_tiny()
    assert tuple(di.q.shape) == (2, 1, 4, 64) and di.seqlens.tolist() == [339, 156]
    assert tuple(di.cache.backing[0].shape) == (132, 2, 16, 2, 64)
    assert tuple(di.block_table.shape) == (2, 66) and di.scale == 1 / 8 and not di.causal


def test_ragged_recipe_at_reduced_size():
    di = I.config_ragged(seed=3, batch=8, max_len=2048, spare_blocks=8)
    bs = 256
    assert tuple(di.q.shape) == (8, 1, 16, 128) and di.cache.block_size == bs
    sl = di.seqlens
    assert bool(((sl >= 1) & (sl <= 2048)).all())
    need = [(n + bs - 1) // bs for n in sl.tolist()]
    assert di.cache.num_blocks == sum(need) + 8
    assert tuple(di.block_table.shape) == (8, 2048 // bs)
    # the blocks a sequence uses are distinct across the batch; columns past
    # its last block point at spare blocks, which are all NaN
    used_ids = torch.cat([di.block_table[b, :k] for b, k in enumerate(need)])
    assert used_ids.unique().numel() == used_ids.numel()
    spare = set(range(di.cache.num_blocks)) - set(used_ids.tolist())
    assert len(spare) == 8
    for b, k in enumerate(need):
        for blk in di.block_table[b, k:].tolist():
            assert blk in spare and torch.isnan(di.cache.k[blk].float()).all()
    used = _used_slots(di.cache, di.block_table, sl)
    assert torch.equal(torch.isnan(di.cache.k.float()).all(-1).all(-1), ~used)


def test_long_context_recipe_at_reduced_size():
    di = I.config_long_context(seed=2, batch=2, seqlen=4096)
    assert tuple(di.q.shape) == (2, 1, 32, 128) and di.seqlens.tolist() == [4096, 4096]
    assert tuple(di.cache.k.shape) == (512, 16, 8, 128) and di.cache.k.is_contiguous()
    assert torch.equal(di.block_table.flatten().sort().values, torch.arange(512, dtype=torch.int32))
    assert di.kv_bytes() == 2 * 4096 * 8 * 128 * 2 * 2


def test_parity_cache_is_empty_and_holds_the_whole_token_stream():
    cache, table, q_all, k_all, v_all = I.config_parity_cache(batch=2, total_tokens=100)
    assert not cache.k.any() and not cache.v.any()
    assert tuple(q_all.shape) == (2, 100, 16, 128) and tuple(k_all.shape) == (2, 100, 4, 128)
    assert table.shape[1] * cache.block_size >= 100
    assert torch.equal(table.flatten().sort().values,
                       torch.arange(cache.num_blocks, dtype=torch.int32))
