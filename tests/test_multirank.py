"""The N>1 benchmark path on CPU: two gloo ranks agree on the max step time and the
summed token count; with weak scaling each rank's adapter set is its own seeded workload, and
with strong scaling the ranks split one adapter set (plora_partition) whose shards together
reproduce the global segment map and, through the oracle, the global weight gradients bit for
bit (no data-path collective)."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    import plora_workloads as wl
    ms = [12.5, 17.25][rank]
    tokens = [1000.0, 3000.0][rank]
    got_max = bench.reduce_max(ms, dist)
    got_sum = bench.reduce_sum(tokens, dist)
    ranks, counts, _ = wl.config3_shape(1003 + 1000 * rank)
    # energy: a rank without a counter reports NaN and the whole-job sum is then NaN on every rank
    e_ok = bench.reduce_sum([4.0, 6.0][rank], dist)
    e_missing = bench.reduce_sum([float("nan"), 6.0][rank], dist)
    q.put((rank, got_max, got_sum, int(counts.sum()), e_ok, e_missing != e_missing))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reductions_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, sm, _, e_ok, e_nan in res:
        assert mx == 17.25 and sm == 4000.0
        assert e_ok == 10.0 and e_nan
    assert res[0][3] != res[1][3]   # each rank draws its own adapter mix


def test_single_process_reductions_are_identity():
    import bench
    assert bench.reduce_max(3.5, None) == 3.5 and bench.reduce_sum(7.0, None) == 7.0


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    import oracle
    import plora_workloads as wl
    g = _global_problem()
    mine = bench.shard_for_rank(g, world, rank)
    o = oracle.weight_grads(mine)
    token_sum = bench.reduce_sum(float(mine.T), dist)
    got = [None] * world
    dist.all_gather_object(got, {"off": mine.off.tolist(), "ranks": mine.ranks.tolist(), "X": mine.X.tobytes(),
                                 "dA": [a.tobytes() for a in o["dA"]], "dB": [b.tobytes() for b in o["dB"]]})
    q.put((rank, token_sum, got))
    dist.barrier()
    dist.destroy_process_group()


def _global_problem():
    import numpy as np
    import plora_workloads as wl
    r = np.array([8, 1, 16, 4, 32, 8, 2, 16, 3])
    return wl.make_problem("shard2", "bf16", 48, 32, r, [40, 0, 300, 7, 120, 65, 1, 90, 33], 2.0 * r,
                           wl.init_llm(48), 91)


def test_two_rank_strong_scaling_shards_gloo():
    import numpy as np
    import oracle
    import packed_lora_fine_b200 as pl
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    g = _global_problem()
    full = oracle.weight_grads(g)
    owner, _ = pl.plora_partition(g.counts, g.ranks, g.d_in, g.d_out, world)
    parts = res[0][2]
    assert res[0][2] == res[1][2]                   # both ranks gathered the same shards
    covered = []
    for part, sh in enumerate(parts):
        ids, local_off, ranges = pl.shard(owner, g.off, part)
        assert sh["off"] == local_off.tolist() and sh["ranks"] == g.ranks[ids].tolist()
        X = np.frombuffer(sh["X"], dtype=g.X.dtype).reshape(-1, g.d_in)
        assert np.array_equal(X, np.concatenate([g.X[a:b] for a, b in ranges]))
        for k, i in enumerate(ids):
            assert np.frombuffer(sh["dA"][k], np.float64).tobytes() == full["dA"][i].tobytes()
            assert np.frombuffer(sh["dB"][k], np.float64).tobytes() == full["dB"][i].tobytes()
        covered += list(ids)
    assert sorted(covered) == list(range(g.n_adapters))
    assert all(ts == float(g.T) for _, ts, _ in res)   # the token sum over ranks is the global count
