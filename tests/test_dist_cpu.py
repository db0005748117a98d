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


def _attn_shard_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle.attention import default_scale, merge_partials, sparse_attention
    from oracle.formats import bf16_to_f64
    from sparse_attention_indexer_lightning_b200 import shard_plan
    from workloads.synth import make_attention
    d = make_attention(5, 8, 900, 120, ragged=100, seed=4)
    lat = bf16_to_f64(d["latent"])
    base, length = shard_plan(lat.shape[0], world)[rank]
    # this rank holds rows [base, base + length): the selection shifted by
    # -base, rows outside its range skipped (another rank's)
    local = d["idx"].astype(np.int64) - base
    local = np.where((d["idx"] >= 0) & (local >= 0) & (local < length), local, -1)
    o, lse = sparse_attention(bf16_to_f64(d["q"]), lat[base:base + length], local, default_scale())
    o_all = [torch.zeros_like(torch.from_numpy(o)) for _ in range(world)]
    l_all = [torch.zeros_like(torch.from_numpy(lse)) for _ in range(world)]
    dist.all_gather(o_all, torch.from_numpy(o))
    dist.all_gather(l_all, torch.from_numpy(lse))
    mo, ml = o_all[0].numpy(), l_all[0].numpy()
    for r in range(1, world):
        mo, ml = merge_partials(mo, ml, o_all[r].numpy(), l_all[r].numpy())
    ro, rl = sparse_attention(bf16_to_f64(d["q"]), lat, d["idx"], default_scale())
    ok = (np.allclose(mo, ro, rtol=1e-12, atol=1e-13) and np.array_equal(np.isneginf(ml), np.isneginf(rl))
          and np.allclose(ml[np.isfinite(rl)], rl[np.isfinite(rl)], rtol=1e-12))
    q.put((rank, bool(ok)))
    dist.destroy_process_group()


def test_history_sharded_attention_merges_to_the_full_attention():
    """Two gloo ranks each hold half of the latent rows, attend over the
    selected rows they hold, all-gather (o, lse) and merge by the
    online-softmax rule: every rank ends with the attention over the whole
    selection (the protocol of the sharded decode, computed by the oracle)."""
    import multiprocessing as mp_
    ctx = mp_.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_attn_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: True, 1: True}
