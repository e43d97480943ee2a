"""gemm_fp8_nt_noalloc — the FP8 GEMM entry point for callers that cannot allocate.

It is called here through the C ABI, as such a caller would, and its output is checked
against the regular gemm_fp8_nt path on the same inputs, on two calls in a row with
different data (the second call reuses the shared scratch the first one left behind).
This file is collected last so a stop-at-first-failure run has already run everything else.
"""

import ctypes

import numpy as np
import pytest

import inputs

from parity import check_gemm, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_scaled_precision_sm_b200 import _lib, ops

    return _lib.load(), ops


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_regular_entry_point_twice(env):
    lib, ops = env
    m, n, k = 384, 672, 1024
    kb = k // 128
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (21, 22):
        p = inputs.dense_fp8_problem(m, n, k, seed=seed)
        A, B = to_dev(p["A"]), to_dev(p["B"])
        sfa, sfb = to_dev(p["sfa"]), to_dev(p["sfb"])  # plain UE8M0 bytes [M, K/128], [N/128, K/128]
        ref = ops.gemm_fp8_nt(A, sfa, B, sfb, sfb_gran_n=128)  # regular path (packs via transform_sf_ue8m0)
        assert ops.device_status() == 0
        D = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        rc = lib.gemm_fp8_nt_noalloc(_vp(A), _vp(sfa), _vp(B), _vp(sfb), _vp(D), _vp(status), m, n, k,
                                     k, k, n, kb, kb, 128, stream)
        assert rc == 0, lib.bsp_status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = D.float().cpu().numpy().astype(np.float64)
        check_gemm(got, ref.float().cpu().numpy().astype(np.float64), f"noalloc call seed {seed}")
        assert torch.equal(D.view(torch.int16), ref.view(torch.int16))  # same kernel, same inputs


def test_noalloc_rejects_scratch_overflow(env):
    lib, _ = env
    buf = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = _vp(buf)
    # packed SFA words for M = 40000 rows at K = 16384 need 64 * 40000 * 2 bytes > 4 MiB
    rc = lib.gemm_fp8_nt_noalloc(p, p, p, p, p, _vp(st), 40000, 128, 16384, 16384, 16384, 128, 128, 128, 128,
                                 None)
    assert rc == -4
