"""The N>1 benchmark path on CPU: two gloo ranks agree on the max step time and the
summed token count, and each rank's adapter set is its own seeded workload (weak scaling,
no data-path collective)."""
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
