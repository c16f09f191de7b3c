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
    """One CP rank on CPU: fp64 partials of its split share (the oracle's),
    written into the library's partial-buffer layout (dist.partials_views:
    fp32 acc [rows][n_local][D] padded to 256 bytes, then (m, l) with m in
    base-2 units), the product exchange (dist.cp_exchange over gloo), then the
    merge's ascending fold over all global splits read back out of the
    gathered rank blocks through the same views."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import math
    import torch
    import oracle
    from paged_kv_decode_31_b200 import inputs as I
    pdist.init("gloo", timeout_s=60)
    split = 64   # small splits so a short context spans several
    B, sq, Hq, Hkv, D = 2, 3, 4, 2, 64
    di = I.p2_case(B, sq, 300, Hq, Hkv, D, 16, causal=True, seed=31, seqlens=[300, 141])
    S = -(-300 // split)
    n_local = -(-S // world)
    begin = rank * n_local
    m, l, acc = oracle.split_partials(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                                      di.scale, True, begin, n_local, split_tokens=split)
    rows = B * sq * Hq
    rank_bytes = pdist.partials_bytes(B, sq, Hq, D, n_local)
    buf = torch.full((rank_bytes,), 0xFF, dtype=torch.uint8)   # unreached partials: garbage
    acc_v, ml_v = pdist.partials_views(buf, B, sq, Hq, D, n_local)
    log2e = 1.0 / math.log(2.0)
    reached = torch.isfinite(m.reshape(rows, n_local))
    acc_v[reached] = acc.reshape(rows, n_local, D)[reached].float()
    ml_v[..., 0][reached] = (m.reshape(rows, n_local)[reached] * log2e).float()
    ml_v[..., 1][reached] = l.reshape(rows, n_local)[reached].float()
    gathered = pdist.cp_exchange(buf, None)
    assert gathered.dtype == torch.uint8 and gathered.numel() == world * rank_bytes
    views = [pdist.partials_views(gathered[r * rank_bytes:(r + 1) * rank_bytes], B, sq, Hq, D,
                                  n_local) for r in range(world)]
    out = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    lse = torch.zeros(B, Hq, sq, dtype=torch.float64)
    for b in range(B):
        n = int(di.seqlens[b])
        for i in range(sq):
            lim = max(min(n, n - sq + i + 1), 0)
            n_s = -(-lim // split)            # the merge reads splits [0, n_s) only
            for h in range(Hq):
                row = (b * sq + i) * Hq + h
                M, Lsum, A = -math.inf, 0.0, torch.zeros(D, dtype=torch.float64)
                for s in range(n_s):          # ascending global split
                    r, ls = divmod(s, n_local)
                    a_v, m_v = views[r]
                    ms, lsv = float(m_v[row, ls, 0]), float(m_v[row, ls, 1])
                    Mn = max(M, ms)
                    ca = 2.0 ** (M - Mn) if M > -math.inf else 0.0
                    cs = 2.0 ** (ms - Mn)
                    Lsum = Lsum * ca + lsv * cs
                    A = A * ca + a_v[row, ls].double() * cs
                    M = Mn
                out[b, i, h] = A / Lsum if Lsum > 0 else 0.0
                lse[b, h, i] = (M + math.log2(Lsum)) * math.log(2.0) if Lsum > 0 else -math.inf
    ro, rl = oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                               di.scale, True)
    ok_out = float((out - ro).abs().max())
    fin = torch.isfinite(rl)
    ok_lse = float((lse[fin] - rl[fin]).abs().max())
    same_empty = bool(torch.equal(torch.isneginf(lse), torch.isneginf(rl)))
    shares = (begin, n_local)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    q.put((rank, ok_out, ok_lse, same_empty, shares, rank_bytes))


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange_and_ascending_merge_with_gloo(world):
    """The split shares cover every split once, in rank order; partial buffers
    in the library's layout go through the product exchange and land side by
    side; folding them in ascending global split order, read through the same
    layout, reproduces the whole-context attention (fp32 partials: 1e-5)."""
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
    for rank, d_out, d_lse, same_empty, shares, rank_bytes in res:
        assert shares == (rank * n_local, n_local)
        assert d_out < 1e-5 and d_lse < 1e-5 and same_empty
    assert pdist.cp_split_share(20000, 2, 3) == (4, 2)


def test_partials_views_match_the_library_size():
    """dist.partials_views describes the buffer pkv_partials_size sizes: the
    (m, l) block ends exactly at the library's byte count, after an acc block
    padded to 256 bytes."""
    import torch
    from paged_kv_decode_31_b200 import binding
    from paged_kv_decode_31_b200 import build as pkv_build
    pkv_build.build()
    for (B, sq, Hq, D, n) in [(2, 3, 4, 64, 3), (4, 1, 32, 128, 32), (1, 7, 6, 64, 1)]:
        need = binding.partials_size(B, sq, Hq, D, n)
        assert pdist.partials_bytes(B, sq, Hq, D, n) == need
        buf = torch.zeros(need, dtype=torch.uint8)
        acc, ml = pdist.partials_views(buf, B, sq, Hq, D, n)
        assert acc.shape == (B * sq * Hq, n, D) and ml.shape == (B * sq * Hq, n, 2)
        assert ml.data_ptr() - buf.data_ptr() == -(-(acc.numel() * 4) // 256) * 256
        assert ml.data_ptr() + ml.numel() * 4 == buf.data_ptr() + need
        with pytest.raises(ValueError):
            pdist.partials_views(buf[:need - 4], B, sq, Hq, D, n)


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
