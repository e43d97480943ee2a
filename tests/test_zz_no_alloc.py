"""gemm_fp8_nt_noalloc — the FP8 GEMM entry point for callers that cannot allocate.

It is called here through the C ABI, as such a caller would, and its output is checked
against the fp64 oracle and against the regular gemm_fp8_nt path on the same inputs, on two
calls in a row with different data (the second call reuses the shared scratch the first one
left behind).  The shapes cover each way the call can run: CTA-pair tiles; the transposed
small-M path with per-row B scales, with its two K halves on one cluster, and with a split
last wave whose partial sums fit in the fixed scratch; and the full 4096 x 7168 x 16384
problem, whose split workspace would not fit, so the last wave runs unsplit.  This file is collected last so a stop-at-first-failure run has
already run everything else.
"""

import ctypes

import numpy as np
import pytest

import inputs

from parity import bf16_to_f64, check_gemm, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SCRATCH_BYTES = 4 << 20  # the fixed device array behind the call


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_scaled_precision_sm_b200 import _lib, ops

    return _lib.load(), ops


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, A, sfa, B, sfb, D, status, m, n, k, gran):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    kb = k // 128
    return lib.gemm_fp8_nt_noalloc(_vp(A), _vp(sfa), _vp(B), _vp(sfb), _vp(D), _vp(status), m, n, k,
                                   A.stride(0), B.stride(0), D.stride(0), sfa.stride(0), sfb.stride(0), gran, stream)


def _split_ws_bytes(plan):
    """fp32 partial sums of a split last wave: one tile-sized slot per slice of each split tile."""
    return plan["split_tiles"] * plan["splits"] * plan["tile_m"] * plan["tile_n"] * 4 if plan["splits"] > 1 else 0


# (M, N, K, sfb_gran_n, path): the path bsp_gemm_plan reports for gemm_fp8_nt, and whether the
# fixed scratch has room for its split workspace
CASES = [
    (384, 672, 1024, 128, "pair, whole tiles"),
    (96, 1000, 1024, 1, "transposed, per-row B scales"),
    (128, 1024, 2048, 1, "transposed, K halves in a cluster"),
    (33, 296, 4096, 1, "transposed, split tail in the fixed scratch"),
    (4096, 7168, 16384, 128, "pair, split workspace too large: unsplit"),
]


@pytest.mark.parametrize("m,n,k,gran,path", CASES)
def test_noalloc_matches_oracle_and_regular_entry_point_twice(env, orc, m, n, k, gran, path):
    lib, ops = env
    plan = ops.gemm_plan("fp8", m, n, k)
    full = m * n > 4_000_000
    if path.startswith("pair"):
        assert plan["transposed"] == 0, plan
    else:
        assert plan["transposed"] == 1, plan
    if "whole" in path:
        assert plan["splits"] == 1, plan
    if "fixed scratch" in path:
        assert plan["splits"] > 1 and not plan["cluster_split"] and _split_ws_bytes(plan) < SCRATCH_BYTES // 2, plan
    if "cluster" in path:
        assert plan["splits"] == 2 and plan["cluster_split"] == 1, plan
    if "too large" in path:
        assert plan["splits"] > 1 and _split_ws_bytes(plan) > SCRATCH_BYTES, plan
    p = inputs.dense_fp8_problem(m, n, k, seed=21, b_block_rows=gran)
    A, B = to_dev(p["A"]), to_dev(p["B"])
    rng = np.random.default_rng(m + n)
    if full:
        rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, 40, replace=False)])).astype(np.int32)
        cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 40, replace=False)])).astype(np.int32)
    for call in range(2):
        # the second call has other scale bytes (and so other products) than the first
        sfa_h = p["sfa"] if call == 0 else (p["sfa"] + rng.integers(-3, 4, p["sfa"].shape)).astype(np.uint8)
        sfb_h = p["sfb"] if call == 0 else (p["sfb"] + rng.integers(-3, 4, p["sfb"].shape)).astype(np.uint8)
        sfa, sfb = to_dev(sfa_h), to_dev(sfb_h)  # plain UE8M0 bytes [M, K/128], [ceil(N/g), K/128]
        ref_gpu = ops.gemm_fp8_nt(A, sfa, B, sfb, sfb_gran_n=gran)  # regular path (packs via transform_sf_ue8m0)
        assert ops.device_status() == 0
        D = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        rc = _noalloc(lib, A, sfa, B, sfb, D, status, m, n, k, gran)
        assert rc == 0, lib.bsp_status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        if full:
            ri, ci = torch.from_numpy(rows).long().cuda(), torch.from_numpy(cols).long().cuda()
            got = bf16_to_f64(D[ri][:, ci])
            ref = orc.gemm_fp8(p["A"], sfa_h, p["B"], sfb_h, gran_n=gran, rows=rows, cols=cols)
            assert not torch.isnan(D).any()
        else:
            got = bf16_to_f64(D)
            ref = orc.gemm_fp8(p["A"], sfa_h, p["B"], sfb_h, gran_n=gran)
        check_gemm(got, ref, f"noalloc {path} call {call}")
        check_gemm(bf16_to_f64(D[:64]) if full else got, bf16_to_f64(ref_gpu[:64]) if full else bf16_to_f64(ref_gpu),
                   f"noalloc vs gemm_fp8_nt, {path} call {call}")
        if "unsplit" not in path:
            # the same plan on the same inputs: the same kernel gives the same bytes
            assert torch.equal(D.view(torch.int16), ref_gpu.view(torch.int16))


def test_noalloc_flags_nan_scale_byte(env):
    # UE8M0 byte 0xFF is NaN: the packing latches BSP_ERR_DEVICE_CHECK in the caller's word
    lib, ops = env
    m, n, k = 256, 448, 512
    p = inputs.dense_fp8_problem(m, n, k, seed=3)
    p["sfa"][17, 2] = 0xFF
    A, B, sfa, sfb = (to_dev(p[x]) for x in ("A", "B", "sfa", "sfb"))
    D = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc(lib, A, sfa, B, sfb, D, status, m, n, k, 128) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == -7
    assert ops.device_status() == 0  # the library's own word is untouched


def test_noalloc_rejects_scratch_overflow(env):
    lib, _ = env
    buf = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = _vp(buf)
    # packed SFA words for M = 40000 rows at K = 16384 need 64 * 40000 * 2 bytes > 4 MiB
    rc = lib.gemm_fp8_nt_noalloc(p, p, p, p, p, _vp(st), 40000, 128, 16384, 16384, 16384, 128, 128, 128, 128,
                                 None)
    assert rc == -4
