"""Multi-rank logic of bench.py on CPU: two gloo ranks, as torchrun would start
them for `bench.py --gpus 2` (replicas, weak scaling)."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank measured a different time; the job time is the slowest rank's
        ms = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world, "cpu")
        q.put((rank, ms, bench.job_tokens_per_s(16, world, ms[0]), bench.rank_seed(0xD5400005, rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_sum_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, tps, seed in res:
        assert ms == [2.0, 5.0]  # element-wise max over ranks
        assert tps == pytest.approx(16 * world / 2.0e-3)  # all ranks' tokens over the slowest time
    seeds = [r[3] for r in res]
    assert len(set(seeds)) == world  # replicas draw distinct inputs


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    assert bench.job_tokens_per_s(1, 1, 0.5) == pytest.approx(2000.0)
