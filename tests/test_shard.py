"""Host logic of the sharded GEMM (block_scaled_precision_sm_b200.shard) on CPU.

The shard arithmetic is checked directly; the all-gather that rebuilds D from the column
shards runs on two and three gloo ranks, each standing in for its GPU's GEMM with a plain
float product of its shard (the GPU tests check the sharded GEMM itself against the oracle).
"""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
mp = pytest.importorskip("torch.multiprocessing")

from block_scaled_precision_sm_b200 import shard  # noqa: E402


@pytest.mark.parametrize("n,world", [(7168, 8), (7168, 3), (300, 2), (100, 4), (4096, 1), (1000, 16)])
def test_n_shard_bounds_cover_n_in_aligned_balanced_blocks(n, world):
    b = shard.n_shard_bounds(n, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == n
    for (a0, a1), (c0, c1) in zip(b, b[1:]):
        assert a1 == c0  # contiguous, no overlap
    for n0, n1 in b:
        assert (n0 % 128 == 0 or n0 == n) and n0 <= n1  # an empty range sits at the end
        assert n1 % 128 == 0 or n1 == n
    widths = [-(-(n1 - n0) // 128) for n0, n1 in b]  # blocks per rank
    assert max(widths) - min(widths) <= 1
    if world <= -(-n // 128):
        assert min(widths) >= 1  # nobody idles while there are blocks to go round


def test_n_shard_bounds_headline_split():
    assert shard.n_shard_bounds(7168, 8) == [(896 * r, 896 * (r + 1)) for r in range(8)]


def test_expert_shard_bounds():
    assert shard.expert_shard_bounds(32, 8) == [(4 * r, 4 * r + 4) for r in range(8)]
    b = shard.expert_shard_bounds(5, 3)
    assert b == [(0, 2), (2, 4), (4, 5)]
    with pytest.raises(ValueError):
        shard.expert_shard_bounds(0, 2)


def test_shard_b_takes_matching_scale_rows():
    n, k = 300, 256
    B = torch.arange(n)[:, None].expand(n, k)
    sfb = torch.arange(-(-n // 128))[:, None].expand(-1, k // 128)
    b1, s1 = shard.shard_b(B, sfb, n, 1, 2, sfb_gran_n=128)
    assert b1[0, 0] == 256 and b1.shape[0] == 44 and s1.shape[0] == 1 and s1[0, 0] == 2
    sfr = torch.arange(n)[:, None].expand(n, 2)
    b0, s0 = shard.shard_b(B, sfr, n, 0, 2, sfb_gran_n=1)
    assert b0.shape[0] == 256 and s0.shape[0] == 256 and s0[-1, 0] == 255


def test_localize_expert_indices():
    idx = torch.tensor([4, 4, -1, 5, 7, -1], dtype=torch.int32)
    assert shard.localize_expert_indices(idx, 8, 2, 4).tolist() == [0, 0, -1, 1, 3, -1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_worker(rank, world, port, m, n, k, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    g = torch.Generator().manual_seed(5)
    A = torch.randn(m, k, generator=g)
    B = torch.randn(n, k, generator=g)  # every rank draws the same full operands
    n0, n1 = shard.n_shard_bounds(n, world)[rank]
    D_local = A @ B[n0:n1].T  # stands in for this rank's GPU GEMM
    D = shard.all_gather_columns(D_local, shard.n_shard_bounds(n, world))
    ok = D.shape == (m, n) and torch.equal(D, torch.cat([A @ B[a:b].T for a, b in shard.n_shard_bounds(n, world)], 1))
    close = torch.allclose(D, A @ B.T, rtol=1e-5, atol=1e-4)
    dist.destroy_process_group()
    q.put((rank, bool(ok), bool(close)))


@pytest.mark.parametrize("world,n", [(2, 300), (3, 700)])
def test_all_gather_columns_rebuilds_d_on_every_rank(world, n):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, 17, n, 64, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(r, True, True) for r in range(world)]
