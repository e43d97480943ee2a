"""GPU parity of the sharded GEMM: every rank's shard against the oracle on its slice.

The runs here have one GPU, so the ranks of a P-way split are computed one after another on
it, each exactly as that rank would compute it on its own GPU (its rows of B and of B's
scales, or its experts and the rows routed to them); no collective is involved.  The
all-gather that joins the shards is checked on CPU ranks (tests/test_shard.py).
"""

import numpy as np
import pytest

import inputs

from parity import bf16_to_f64, check_gemm, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_scaled_precision_sm_b200 import ops, shard

    assert ops.device_status() == 0
    return ops, shard


@pytest.mark.parametrize("m,n,k,world,gran", [(256, 1000, 1024, 2, 128), (300, 7168, 1024, 8, 128),
                                              (96, 2000, 2048, 3, 1), (512, 640, 512, 8, 1)])
def test_n_sharded_each_rank_matches_its_columns(env, orc, m, n, k, world, gran):
    ops, shard = env
    p = inputs.dense_fp8_problem(m, n, k, seed=m + world, b_block_rows=gran)
    A, sfa = to_dev(p["A"]), to_dev(p["sfa"])
    B, sfb = torch.from_numpy(p["B"]), torch.from_numpy(p["sfb"])
    pieces = []
    for rank, (n0, n1) in enumerate(shard.n_shard_bounds(n, world)):
        b, s = shard.shard_b(B, sfb, n, rank, world, sfb_gran_n=gran)
        D = shard.gemm_fp8_nt_n_sharded(A, sfa, to_dev(b.numpy()), to_dev(s.numpy()), n, rank, world,
                                        sfb_gran_n=gran)
        assert ops.device_status() == 0
        assert tuple(D.shape) == (m, n1 - n0)
        if n1 == n0:
            continue
        cols = np.arange(n0, n1, dtype=np.int32)
        ref = orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=gran, cols=cols)
        got = bf16_to_f64(D)
        if got.size >= 1000:
            check_gemm(got, ref, f"rank {rank}/{world} columns [{n0}, {n1})")
        pieces.append(got)
    full = np.concatenate(pieces, axis=1)
    check_gemm(full, orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=gran), f"all shards, {world} ranks")


@pytest.mark.parametrize("world", [2, 4])
def test_expert_sharded_grouped_each_rank(env, orc, world):
    ops, shard = env
    counts = [100, 0, 150, 50, 300, 20, 128, 77]
    n, k = 448, 512
    p = inputs.grouped_fp8_problem(len(counts), sum(counts), n, k, seed=3, counts=counts)
    idx = p["m_indices"]
    ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], idx)
    # rows routed to rank r: the padded segments of its experts (contiguous in this layout)
    for rank, (g0, g1) in enumerate(shard.expert_shard_bounds(len(counts), world)):
        seg = np.isin(idx, np.arange(g0, g1))
        pad_owner = np.maximum.accumulate(np.where(idx >= 0, idx, -1))  # padding belongs to the expert before it
        rows = np.where(seg | ((idx < 0) & (pad_owner >= g0) & (pad_owner < g1)))[0]
        if rows.size == 0:
            continue
        local_idx = shard.localize_expert_indices(to_dev(idx[rows]), len(counts), rank, world)
        D = shard.m_grouped_gemm_fp8_nt_expert_sharded(
            to_dev(p["A"][rows]), to_dev(p["sfa"][rows]), to_dev(p["B"][g0:g1]), to_dev(p["sfb"][g0:g1]),
            local_idx, len(counts), rank, world)
        assert ops.device_status() == 0
        got = bf16_to_f64(D)
        check_gemm(got, ref[rows], f"experts [{g0}, {g1}) of {len(counts)}")
        assert np.all(got[idx[rows] < 0] == 0.0)
