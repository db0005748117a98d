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
