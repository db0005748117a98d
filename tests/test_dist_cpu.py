"""Multi-process host logic of the benchmark on CPU: two gloo ranks run the
same plumbing bench.py uses under torchrun (barrier, max over ranks, the
weak-scaling aggregate).  The data path has no collective (each rank selects
its own sequences), so this is all the N > 1 path adds."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    w, r, _ = bench.dist_setup(world, backend="gloo")
    bench.barrier(w)
    t = bench.max_over_ranks(1.5 + r, w)          # rank 1 is the slowest
    v = bench.weak_scaling_value(1000.0, t, w)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, t, v))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_agree_on_max_time(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, t, v in out:
        assert w == world
        assert t == 1.5 + (world - 1)
        assert v == pytest.approx(world * 1000.0 / (t * 1e-3))


def _shard_worker(rank, world, port, n_keys, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from sparse_attention_indexer_lightning_b200 import shard_plan
    base, length = shard_plan(n_keys, world)[rank]
    mine = torch.tensor([base, length], dtype=torch.int64)
    got = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(got, mine)
    q.put((rank, [tuple(int(x) for x in g) for g in got]))
    dist.destroy_process_group()


@pytest.mark.parametrize("n_keys", [1019, 32768])
def test_history_shards_cover_the_history_once(n_keys):
    """Each of two gloo ranks takes its history shard; gathered, the shards
    tile [0, n_keys) contiguously with no overlap."""
    import multiprocessing as mp
    import socket
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, n_keys, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = res[0]
    assert res[1] == shards
    pos = 0
    for base, length in shards:
        assert base == pos and length > 0
        pos += length
    assert pos == n_keys
