"""Seeded synthetic inputs for paged-KV attention.

This module is shared by the tests, the bench and the smoke check; it feeds
both the CUDA path and the CPU oracle.  It holds no attention arithmetic: only
random numbers, cache layouts, block tables and sequence lengths.

The recipe follows the aiter test "test(triton/decode): pin non-contiguous
paged KV block stride" (helper _generate_interleaved_block_kvcache and
test_flash_attn_kvcache_noncontiguous_paged):

* q, K and V are bf16 draws from N(0, 1);
* num_blocks = ceil(seqlen_k / block_size) * batch * 3 (three-fold
  over-allocation, so that a random permutation scatters each sequence's
  blocks over the whole pool);
* block_table = randperm(num_blocks) reshaped to (batch, num_blocks / batch);
* the interleaved cache is one [num_blocks, 2, block_size, Hkv, D] buffer whose
  K = [:, 0] and V = [:, 1] views are non-contiguous with block stride
  2 * block_size * Hkv * D; the contiguous cache is two
  [num_blocks, block_size, Hkv, D] buffers;
* cache_seqlens are uniform integers in [1, seqlen_k] unless fixed.

Two additions that guard against over-reads: slots past a sequence's length in
its last block, and blocks no sequence references, can be filled with NaN, and
table entries past a sequence's last used block can point at NaN spare blocks.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

BF16 = torch.bfloat16


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """N(0,1) draws rounded to bf16 (drawn in fp32 on the generator's device)."""
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(BF16)


@dataclass
class PagedCache:
    """A paged KV cache plus the views the library and the oracle consume."""
    k: torch.Tensor              # [num_blocks, block_size, Hkv, D] view (maybe non-contiguous)
    v: torch.Tensor              # same shape as k
    backing: Sequence[torch.Tensor]  # the buffers the views live in
    layout: str                  # "contiguous" | "interleaved"

    @property
    def num_blocks(self) -> int:
        return int(self.k.shape[0])

    @property
    def block_size(self) -> int:
        return int(self.k.shape[1])

    def to(self, device) -> "PagedCache":
        if self.layout == "interleaved":
            kv = self.backing[0].to(device)
            return PagedCache(kv[:, 0], kv[:, 1], (kv,), self.layout)
        k = self.backing[0].to(device)
        v = self.backing[1].to(device)
        return PagedCache(k, v, (k, v), self.layout)

    def clone(self) -> "PagedCache":
        """A deep copy with the same layout (same device)."""
        if self.layout == "interleaved":
            kv = self.backing[0].clone()
            return PagedCache(kv[:, 0], kv[:, 1], (kv,), self.layout)
        k, v = self.k.clone(), self.v.clone()
        return PagedCache(k, v, (k, v), self.layout)

    def as_contiguous(self) -> "PagedCache":
        """The same data in a contiguous two-buffer layout (bitwise copy)."""
        k = self.k.contiguous().clone()
        v = self.v.contiguous().clone()
        return PagedCache(k, v, (k, v), "contiguous")


def make_cache(num_blocks: int, block_size: int, Hkv: int, D: int, layout: str,
               gen: torch.Generator, device="cpu") -> PagedCache:
    if layout == "interleaved":
        kv = randn_bf16((num_blocks, 2, block_size, Hkv, D), gen, device)
        return PagedCache(kv[:, 0], kv[:, 1], (kv,), layout)
    if layout == "contiguous":
        k = randn_bf16((num_blocks, block_size, Hkv, D), gen, device)
        v = randn_bf16((num_blocks, block_size, Hkv, D), gen, device)
        return PagedCache(k, v, (k, v), layout)
    raise ValueError(f"unknown layout {layout!r}")


def randperm_table(num_blocks: int, batch: int, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """randperm(num_blocks) reshaped to (batch, num_blocks // batch), int32."""
    assert num_blocks % batch == 0
    perm = torch.randperm(num_blocks, generator=gen, device=device, dtype=torch.int64)
    return perm.to(torch.int32).reshape(batch, num_blocks // batch)


def uniform_seqlens(batch: int, lo: int, hi: int, gen: torch.Generator) -> torch.Tensor:
    """Integers uniform in [lo, hi], int32 (CPU)."""
    return torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64).to(torch.int32)


def poison_unused(cache: PagedCache, block_table: torch.Tensor, seqlens: torch.Tensor) -> None:
    """Fill with NaN every slot the sequences do not use: slots past seqlens[b]
    in a sequence's last block and every block no sequence references within
    its length.  Works in place on the cache's backing buffers (any device)."""
    bs = cache.block_size
    used = torch.zeros(cache.num_blocks, dtype=torch.bool)
    bt = block_table.cpu()
    nan = float("nan")
    for b, n in enumerate(seqlens.cpu().tolist()):
        nblk = (n + bs - 1) // bs
        ids = bt[b, :nblk].to(torch.int64)
        used[ids] = True
        if n % bs and nblk > 0:
            last = int(bt[b, nblk - 1])
            cache.k[last, n % bs:] = nan
            cache.v[last, n % bs:] = nan
    unused = (~used).nonzero().flatten().to(cache.k.device)
    if unused.numel():
        cache.k[unused] = nan
        cache.v[unused] = nan


@dataclass
class DecodeInputs:
    """Everything one decode / prefill call takes, on one device."""
    q: torch.Tensor              # [B, sq, Hq, D] bf16
    cache: PagedCache
    block_table: torch.Tensor    # [B, nblk] int32
    seqlens: torch.Tensor        # [B] int32
    Hq: int
    Hkv: int
    D: int
    scale: float
    causal: bool
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])

    @property
    def seqlen_q(self) -> int:
        return int(self.q.shape[1])

    def to(self, device) -> "DecodeInputs":
        return DecodeInputs(self.q.to(device), self.cache.to(device),
                            self.block_table.to(device), self.seqlens.to(device),
                            self.Hq, self.Hkv, self.D, self.scale, self.causal,
                            dict(self.extra))

    def kv_bytes(self) -> int:
        """Algorithmic KV bytes: every visible token read once per KV head, K and V, bf16."""
        return int(self.seqlens.to(torch.int64).sum().item()) * self.Hkv * self.D * 2 * 2


def p2_case(batch: int, seqlen_q: int, seqlen_k: int, Hq: int, Hkv: int, D: int,
            block_size: int, causal: bool, layout: str = "interleaved", seed: int = 0,
            seqlens: Optional[Sequence[int]] = None, poison: bool = False,
            scale: Optional[float] = None, device="cpu") -> DecodeInputs:
    """One case of the aiter non-contiguous paged test grid (see module doc)."""
    gen = _gen(seed)
    q = randn_bf16((batch, seqlen_q, Hq, D), gen)
    num_blocks = math.ceil(seqlen_k / block_size) * batch * 3
    cache = make_cache(num_blocks, block_size, Hkv, D, layout, gen)
    table = randperm_table(num_blocks, batch, gen)
    if seqlens is None:
        sl = uniform_seqlens(batch, 1, seqlen_k, gen)
    else:
        sl = torch.tensor(list(seqlens), dtype=torch.int32)
    if poison:
        poison_unused(cache, table, sl)
    sc = (1.0 / math.sqrt(D)) if scale is None else float(scale)
    di = DecodeInputs(q, cache, table, sl, Hq, Hkv, D, sc, causal)
    return di.to(device) if str(device) != "cpu" else di


# ----------------------------------------------------------------------------
# The five workloads the library is measured and checked on.
# ----------------------------------------------------------------------------

def config_tiny(seed: int = 0, device="cpu") -> DecodeInputs:
    """Tiny paged decode: batch 2, seqlen_q 1, contexts {339, 156}, Hq 4 / Hkv 2,
    D 64, block_size 16, interleaved [132, 2, 16, 2, 64], randperm table [2, 66],
    scale 1/8, non-causal."""
    return p2_case(2, 1, 339, 4, 2, 64, 16, causal=False, layout="interleaved",
                   seed=seed, seqlens=[339, 156], scale=1.0 / 8.0, device=device)


def config_gqa_shard(seed: int = 0, device="cpu") -> DecodeInputs:
    """GQA decode shard: batch 32, seqlen_q 1, every context 4096, Hq 32 / Hkv 8,
    D 128, contiguous cache, block_size 16, 3x over-allocated randperm table."""
    return p2_case(32, 1, 4096, 32, 8, 128, 16, causal=False, layout="contiguous",
                   seed=seed, seqlens=[4096] * 32, device=device)


def config_ragged(seed: int = 0, device="cpu", batch: int = 64, max_len: int = 32768,
                  spare_blocks: int = 64) -> DecodeInputs:
    """Ragged decode: batch 64, seqlen_q 1, contexts uniform in [1, 32768],
    Hq 16 / Hkv 4, D 128, interleaved [num_blocks, 2, 256, 4, 128], block_size
    256.  num_blocks = sum(ceil(len / 256)) + spare; table entries past each
    sequence's last block point at spare blocks; every unused slot and every
    spare block is NaN, so an over-read poisons the output."""
    gen = _gen(seed)
    Hq, Hkv, D, bs = 16, 4, 128, 256
    sl = uniform_seqlens(batch, 1, max_len, gen)
    need = [(n + bs - 1) // bs for n in sl.tolist()]
    width = (max_len + bs - 1) // bs
    num_blocks = sum(need) + spare_blocks
    q = randn_bf16((batch, 1, Hq, D), gen, device)
    cache = make_cache(num_blocks, bs, Hkv, D, "interleaved", gen, device)
    perm = torch.randperm(num_blocks, generator=gen, dtype=torch.int64).to(torch.int32)
    table = torch.empty(batch, width, dtype=torch.int32)
    used_ids, spare = perm[: sum(need)], perm[sum(need):]
    off = 0
    for b, k in enumerate(need):
        table[b, :k] = used_ids[off: off + k]
        off += k
        rest = width - k
        if rest:
            table[b, k:] = spare[torch.arange(rest) % spare_blocks]
    poison_unused(cache, table, sl)
    return DecodeInputs(q, cache, table.to(device), sl.to(device), Hq, Hkv, D,
                        1.0 / math.sqrt(D), False)


def config_long_context(seed: int = 0, device="cpu", batch: int = 4,
                        seqlen: int = 131072) -> DecodeInputs:
    """Long-context split-K decode: batch 4, seqlen_q 1, contexts 131072,
    Hq 32 / Hkv 8, D 128, block_size 16, contiguous cache, randperm table
    [4, 8192] (num_blocks = 32768, 2.147 GB of K+V)."""
    gen = _gen(seed, device)
    Hq, Hkv, D, bs = 32, 8, 128, 16
    nblk = seqlen // bs
    num_blocks = nblk * batch
    q = randn_bf16((batch, 1, Hq, D), gen, device)
    cache = make_cache(num_blocks, bs, Hkv, D, "contiguous", gen, device)
    table = randperm_table(num_blocks, batch, gen, device)
    sl = torch.full((batch,), seqlen, dtype=torch.int32, device=device)
    return DecodeInputs(q, cache, table, sl, Hq, Hkv, D, 1.0 / math.sqrt(D), False)


def config_parity_cache(seed: int = 0, batch: int = 8, total_tokens: int = 2048 + 64 + 17,
                        device="cpu"):
    """The prefill/decode parity workload's empty cache and token stream:
    Hq 16 / Hkv 4, D 128, block_size 16, batch 8, capacity for the 2048-token
    prefill, 64 decode steps and a 17-token multi-query step.  Returns
    (cache, table, q_all [B, T, Hq, D], k_all, v_all [B, T, Hkv, D])."""
    gen = _gen(seed)
    Hq, Hkv, D, bs = 16, 4, 128, 16
    nblk = math.ceil(total_tokens / bs) * 3
    num_blocks = nblk * batch
    cache = make_cache(num_blocks, bs, Hkv, D, "contiguous", gen)
    cache.k.zero_()
    cache.v.zero_()
    table = randperm_table(num_blocks, batch, gen)
    q_all = randn_bf16((batch, total_tokens, Hq, D), gen)
    k_all = randn_bf16((batch, total_tokens, Hkv, D), gen)
    v_all = randn_bf16((batch, total_tokens, Hkv, D), gen)
    if str(device) != "cpu":
        cache = cache.to(device)
        table, q_all, k_all, v_all = (t.to(device) for t in (table, q_all, k_all, v_all))
    return cache, table, q_all, k_all, v_all
