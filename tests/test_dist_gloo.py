"""Multi-rank host logic on CPU: world size 2 over the gloo backend."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from paged_kv_decode_31_b200 import dist as pdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    r, w, lr = pdist.rank_env()
    pdist.init("gloo", timeout_s=60)
    got = pdist.max_over_ranks(10.0 * (rank + 1))
    sh = list(pdist.shard(9, r, w))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, r, w, lr, got, sh))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_shards_with_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[4] for o in out] == [10.0 * world] * world          # max over ranks on every rank
    assert [o[1] for o in out] == list(range(world)) and all(o[2] == world for o in out)
    shards = [o[5] for o in out]
    assert sorted(x for s in shards for x in s) == list(range(9))  # disjoint cover


def test_shard_sizes_and_rate():
    for n in range(0, 20):
        for w in range(1, 5):
            parts = [pdist.shard(n, r, w) for r in range(w)]
            sizes = [len(p) for p in parts]
            assert sum(sizes) == n and max(sizes) - min(sizes) <= 1
            assert [x for p in parts for x in p] == list(range(n))
    assert pdist.weak_scaling_rate(100.0, 4, 10, 1000.0) == 4000.0
    assert pdist.max_over_ranks(3.5) == 3.5                          # no process group


def _cp_worker(rank, world, port, q):
    """One CP rank on CPU: fp64 partials of its split share (the oracle's), the
    gloo exchange of the packed buffers, then the ascending fold over all
    global splits from the gathered blocks."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import math
    import torch
    import torch.distributed as dist
    import oracle
    from paged_kv_decode_31_b200 import inputs as I
    pdist.init("gloo", timeout_s=60)
    split = 64   # small splits so a short context spans several
    di = I.p2_case(2, 3, 300, 4, 2, 64, 16, causal=True, seed=31, seqlens=[300, 141])
    S = -(-300 // split)
    n_local = -(-S // world)
    begin = rank * n_local
    m, l, acc = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                      di.scale, True, begin, n_local, split_tokens=split)
    block = torch.cat([acc.reshape(-1), m.reshape(-1), l.reshape(-1)])
    gathered = pdist.cp_exchange(block, None).reshape(world, -1)
    B, sq, Hq, D = di.q.shape
    na = B * sq * Hq * n_local * D
    nm = B * sq * Hq * n_local
    out = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    lse = torch.zeros(B, Hq, sq, dtype=torch.float64)
    for b in range(B):
        for i in range(sq):
            for h in range(Hq):
                M, Lsum, A = -math.inf, 0.0, torch.zeros(D, dtype=torch.float64)
                for s in range(world * n_local):          # ascending global split
                    r, ls = divmod(s, n_local)
                    blk = gathered[r]
                    idx = ((b * sq + i) * Hq + h) * n_local + ls
                    ms, lsv = float(blk[na + idx]), float(blk[na + nm + idx])
                    if ms == -math.inf:
                        continue
                    a_s = blk[idx * D:(idx + 1) * D]
                    Mn = max(M, ms)
                    ca, cs = math.exp(M - Mn) if M > -math.inf else 0.0, math.exp(ms - Mn)
                    Lsum = Lsum * ca + lsv * cs
                    A = A * ca + a_s * cs
                    M = Mn
                out[b, i, h] = A / Lsum if Lsum > 0 else 0.0
                lse[b, h, i] = M + math.log(Lsum) if Lsum > 0 else -math.inf
    ro, rl = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                               di.scale, True)
    ok_out = float((out - ro).abs().max())
    fin = torch.isfinite(rl)
    ok_lse = float((lse[fin] - rl[fin]).abs().max())
    same_empty = bool(torch.equal(torch.isneginf(lse), torch.isneginf(rl)))
    shares = (begin, n_local)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ok_out, ok_lse, same_empty, shares))


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange_and_ascending_merge_with_gloo(world):
    """The split shares cover every split once, in rank order; the exchanged
    blocks land side by side; folding them in ascending global split order
    reproduces the whole-context attention (fp64, CPU)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    S = -(-300 // 64)
    n_local = -(-S // world)
    for rank, d_out, d_lse, same_empty, shares in res:
        assert shares == (rank * n_local, n_local)
        assert d_out < 1e-12 and d_lse < 1e-12 and same_empty
    assert pdist.cp_split_share(20000, 2, 3) == (4, 2)


@pytest.mark.parametrize("ctx,world", [(1, 1), (4096, 1), (4097, 2), (20000, 3), (8192, 8), (0, 4)])
def test_cp_shares_cover_every_split_once_in_rank_order(ctx, world):
    """Contiguous equal shares of the S = ceil(ctx / 4096) splits (S >= 1): every
    split belongs to exactly one rank, rank r's share starts where rank r-1's
    ends, and shares past S only happen at the end (more ranks than splits)."""
    S = max(1, -(-ctx // 4096))
    shares = [pdist.cp_split_share(ctx, r, world) for r in range(world)]
    n = shares[0][1]
    assert all(nl == n for _, nl in shares) and n >= 1
    assert [b for b, _ in shares] == [r * n for r in range(world)]
    covered = [s for b, nl in shares for s in range(b, b + nl) if s < S]
    assert covered == list(range(S))
