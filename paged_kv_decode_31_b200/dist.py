"""Host-side multi-process helpers (one process per GPU, torch.distributed).

The decode path partitions into independent (sequence, KV head, split) units,
so ranks shard sequences and need no collective on the data path; the only
collectives are the timing barrier and the max-over-ranks reduction of the
timed region.  Context parallelism over one long context has one exchange
step: each rank computes the partials of its contiguous share of the 4096-token
splits, the partial buffers are all-gathered, and every rank runs the same
ascending-split merge (RL-Kernel PR #284 "feat(attention): add CP backward
drift validation", Changes: CP world size, KV chunk size, fixed
global_block_index merge order).  Everything here also runs on the `gloo`
backend on CPU.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def rank_env() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 120) -> None:
    """Initialise the default process group with a short timeout, so ranks
    that wait for a missing peer fail instead of hanging."""
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def shard(n_items: int, rank: int, world: int) -> range:
    """Contiguous share of n_items for this rank (sizes differ by at most 1)."""
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return units_per_rank * world * steps / (max_ms / 1e3)


SPLIT_TOKENS = 4096


def cp_split_share(max_seqlen_k: int, rank: int, world: int) -> Tuple[int, int]:
    """(split_begin, n_splits_local) of this rank: the S = ceil(max_seqlen_k /
    4096) splits cut into `world` contiguous blocks of n_local = ceil(S / world)
    splits (the last blocks may run past S; their extra splits see no key)."""
    S = max(1, -(-int(max_seqlen_k) // SPLIT_TOKENS))
    n_local = -(-S // world)
    return rank * n_local, n_local


def partials_bytes(batch: int, seqlen_q: int, Hq: int, D: int, n_splits_local: int) -> int:
    """Bytes of one rank's partial buffer (what pkv_partials_size returns),
    computed on the host without the library: see partials_views."""
    rows = batch * seqlen_q * Hq
    return -(-(rows * n_splits_local * D * 4) // 256) * 256 + rows * n_splits_local * 2 * 4


def partials_views(buf: torch.Tensor, batch: int, seqlen_q: int, Hq: int, D: int,
                   n_splits_local: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """The two arrays inside one rank's partial buffer (a uint8 tensor of
    partials_size(batch, seqlen_q, Hq, D, n_splits_local) bytes, the layout
    pkv_paged_attn_partials writes and pkv_merge_partials reads): acc fp32
    [rows, n_local, D], then, after padding to a multiple of 256 bytes, (m, l)
    fp32 [rows, n_local, 2], rows = batch * seqlen_q * Hq in (b, i, h) order.
    m is the split's max score in base-2 units (scale * log2(e) * q.k), l the
    sum of 2^(s - m) and acc the sum of 2^(s - m) v over the split's visible
    keys.  Views, not copies; usable on any device."""
    rows = batch * seqlen_q * Hq
    acc_bytes = -(-(rows * n_splits_local * D * 4) // 256) * 256
    need = partials_bytes(batch, seqlen_q, Hq, D, n_splits_local)
    flat = buf.reshape(-1)
    if flat.dtype != torch.uint8 or flat.numel() < need:
        raise ValueError(f"partial buffer must be uint8 with at least {need} bytes")
    acc = flat[:rows * n_splits_local * D * 4].view(torch.float32).view(rows, n_splits_local, D)
    ml = flat[acc_bytes:need].view(torch.float32).view(rows, n_splits_local, 2)
    return acc, ml


def cp_exchange(partials: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's partial buffer (equal sizes) side by side, rank
    0's first: the layout pkv_merge_partials reads.  Every rank takes this
    collective step, whatever the world size."""
    world = dist.get_world_size(group)
    flat = partials.reshape(-1)
    if dist.get_backend(group) == "nccl":
        out = torch.empty(world * flat.numel(), dtype=flat.dtype, device=flat.device)
        dist.all_gather_into_tensor(out, flat, group=group)
        return out
    parts = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(parts, flat, group=group)
    return torch.cat(parts)


def cp_attention(q, k_cache, v_cache, block_table, seqlens, max_seqlen_k, *, scale=None,
                 causal=False, group=None):
    """Context-parallel attention on this rank: partials of its split share,
    the exchange, and the merge.  Every rank returns the same (out, lse), bitwise
    those of one paged_decode_attn call over the whole context.  This rank's
    cache and block table need only hold the tokens of its splits."""
    from . import binding
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    begin, n_local = cp_split_share(max_seqlen_k, rank, world)
    part = binding.paged_attn_partials(q, k_cache, v_cache, block_table, seqlens, begin, n_local,
                                       scale=scale, causal=causal)
    gathered = cp_exchange(part, group)
    return binding.merge_partials(gathered, world, n_local, seqlens, tuple(q.shape),
                                  causal=causal)
