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
