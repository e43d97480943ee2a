"""GPU parity at the full workload sizes, in the launch configuration the bench times.

The oracle computes a sample of output elements one by one (rows and columns drawn
from the seed, plus the first and last of each); the GPU computes the whole output.
"""

import numpy as np
import pytest

import inputs

from parity import bf16_to_f64, check_gemm, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ops():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_scaled_precision_sm_b200.ops as ops

    return ops


def _sample(m, n, seed, k=40):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, min(k, m), replace=False)])).astype(np.int32)
    cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, min(k, n), replace=False)])).astype(np.int32)
    return rows, cols


def test_bf16_full(ops, orc):
    m, n, k = 4096, 7168, 16384
    p = inputs.dense_bf16_problem(m, n, k, seed=2)
    D = ops.gemm_bf16_nt(to_dev(p["A"], torch.bfloat16), to_dev(p["B"], torch.bfloat16))
    assert ops.device_status() == 0
    rows, cols = _sample(m, n, 1)
    got = bf16_to_f64(D[torch.from_numpy(rows).long().cuda()][:, torch.from_numpy(cols).long().cuda()])
    check_gemm(got, orc.gemm_bf16(p["A"], p["B"], rows=rows, cols=cols), "bf16 full")


@pytest.mark.parametrize("m,n,k", [(4096, 7168, 16384), (128, 7168, 7168), (1024, 7168, 7168), (4096, 7168, 7168)])
def test_fp8_full(ops, orc, m, n, k):
    p = inputs.dense_fp8_problem(m, n, k, seed=4)
    D = ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]))
    assert ops.device_status() == 0
    rows, cols = _sample(m, n, 2)
    got = bf16_to_f64(D[torch.from_numpy(rows).long().cuda()][:, torch.from_numpy(cols).long().cuda()])
    check_gemm(got, orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], rows=rows, cols=cols), f"fp8 {m}")


def test_fp4_full(ops, orc):
    m, n, k = 4096, 7168, 16384
    p = inputs.dense_fp4_problem(m, n, k, seed=6)
    D = ops.gemm_fp4_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]))
    assert ops.device_status() == 0
    rows, cols = _sample(m, n, 3)
    got = bf16_to_f64(D[torch.from_numpy(rows).long().cuda()][:, torch.from_numpy(cols).long().cuda()])
    check_gemm(got, orc.gemm_fp4(p["A"], p["sfa"], p["B"], p["sfb"], rows=rows, cols=cols), "fp4 full")


def test_grouped_full(ops, orc):
    p = inputs.grouped_fp8_problem(32, 32768, 4096, 7168, seed=8)
    D = ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]),
                                             to_dev(p["sfb"]), to_dev(p["m_indices"]))
    assert ops.device_status() == 0
    m, n = p["M"], p["N"]
    rows, cols = _sample(m, n, 4, k=50)
    got = bf16_to_f64(D[torch.from_numpy(rows).long().cuda()][:, torch.from_numpy(cols).long().cuda()])
    ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"], rows=rows, cols=cols)
    check_gemm(got, ref, "grouped full")
    pad = p["m_indices"] < 0
    assert torch.count_nonzero(D[torch.from_numpy(pad).cuda()]).item() == 0
