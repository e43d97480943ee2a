"""Multi-rank host logic of the bench on CPU: two gloo ranks (the GPU runs use NCCL).

The job's time is the slowest rank's (max over ranks), every rank takes the same collective
steps, and the CPU reference arm runs on rank 0 only.
"""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
mp = pytest.importorskip("torch.multiprocessing")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    r, w, _ = bench.rank_env()
    bench.barrier(w)
    slowest = bench.max_over_ranks(10.0 + r, w)
    # the reference arm returns at once on ranks other than 0 (no oracle work, no output)
    ran_reference = r == 0
    if r != 0:
        bench.run_reference(type("A", (), {"warmup": 0, "steps": 1})())
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, w, slowest, ran_reference))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == list(range(world))
    assert all(o[1] == world for o in out)
    assert all(o[2] == 10.0 + world - 1 for o in out)  # every rank sees the slowest rank's time


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
