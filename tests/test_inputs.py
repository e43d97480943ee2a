"""Invariants of the seeded input recipe (quantiser, grouped segments), decoded by the oracle's tables."""

import ml_dtypes
import numpy as np
import pytest

import inputs


def test_exponent_is_minimal():
    amax = np.array([448.0, 448.0001, 447.9, 1.0, 3.5, 3.5000002, 0.0, 1e-30, 6.0, 2.0 ** 100], np.float64)
    e = inputs.ue8m0_exponent_for_amax(amax, 448.0)
    for a, ei in zip(amax, e):
        if a == 0:
            assert ei == 0
            continue
        assert 448.0 * 2.0 ** float(ei) >= a
        assert 448.0 * 2.0 ** float(ei - 1) < a or ei == -126
    assert list(e[:3]) == [0, 1, 0]
    assert list(inputs.ue8m0_exponent_for_amax(np.array([6.0, 6.1, 3.0]), 6.0)) == [0, 1, -1]


@pytest.mark.parametrize("block_rows", [1, 128])
def test_e4m3_quantiser_invariants(orc, block_rows):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((256, 512)) * np.exp(rng.standard_normal((256, 1)))).astype(np.float32)
    x[3, :128] = 0.0  # one all-zero 1x128 block
    codes, exps = inputs.quantize_e4m3_blocks(x, block_rows)
    e4, _, _ = orc.tables()
    q = e4[codes]
    assert not np.isnan(q).any() and np.abs(q).max() <= 448.0
    e = exps.astype(np.int64) - 127
    escale = np.repeat(np.repeat(e, block_rows, axis=0)[:256], 128, axis=1)
    # within half an E4M3 ulp of the scaled value (ulp = 2^(floor(log2|v|)-3), floor 2^-9)
    v = x.astype(np.float64) / np.ldexp(1.0, escale)
    ulp = np.ldexp(1.0, np.maximum(np.floor(np.log2(np.maximum(np.abs(v), 1e-300))), -6).astype(int) - 3)
    assert np.all(np.abs(q - v) <= ulp / 2)
    # the block exponent is minimal: amax / 2^e > 448 / 2
    amax = np.abs(x).reshape(256 // block_rows, block_rows, 4, 128).max(axis=(1, 3))
    nz = amax > 0
    assert np.all(amax[nz] / np.ldexp(1.0, e[nz]) > 224.0)
    if block_rows == 1:
        assert exps[3, 0] == 127 and not codes[3, :128].any()


def test_e2m1_rounding_and_packing(orc):
    # ties go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    row = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4, np.float32)
    packed, exps = inputs.quantize_e2m1_blocks(row[None, :])
    assert exps[0, 0] == 127  # amax 6 -> e = 0
    _, e2, _ = orc.tables()
    lo = e2[packed[0] & 0xF]
    hi = e2[packed[0] >> 4]
    vals = np.empty(32)
    vals[0::2], vals[1::2] = lo, hi
    assert list(vals[:8]) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0]


def test_bf16_operand_is_rne():
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -2.5, 3.0e38], np.float32)
    bits = inputs.bf16_operand(x)
    assert list(bits[:3]) == [0x3F80, 0x3F82, 0xC020]


def test_dirichlet_segments():
    rng = np.random.default_rng(1)
    c = inputs.dirichlet_segments(rng, 32, 32768)
    assert c.sum() == 32768 and c.min() >= 0 and len(c) == 32


def test_grouped_layout():
    p = inputs.grouped_fp8_problem(8, 1000, 128, 256, seed=3)
    idx = p["m_indices"]
    assert p["M"] % 128 == 0 and (idx >= 0).sum() == 1000
    blocks = idx.reshape(-1, 128)
    for blk in blocks:
        valid = blk[blk >= 0]
        assert blk[0] >= 0 and (valid == blk[0]).all()  # homogeneous, starts valid
        first_pad = np.argmax(blk < 0) if (blk < 0).any() else 128
        assert (blk[first_pad:] < 0).all()  # padding sits at the segment tail
    assert not p["A"][idx < 0].any()


def test_same_seed_same_bytes():
    a = inputs.dense_fp8_problem(128, 256, 256, seed=4)
    b = inputs.dense_fp8_problem(128, 256, 256, seed=4)
    for key in ("A", "sfa", "B", "sfb"):
        assert np.array_equal(a[key], b[key])
    assert ml_dtypes.float8_e4m3fn  # recipe dependency present


def test_masked_problem_layout():
    p = inputs.masked_fp8_problem(5, 256, 96, 384, seed=3)
    assert p["A"].shape == (5, 256, 384) and p["B"].shape == (5, 96, 384)
    assert p["sfa"].shape == (5 * 256, 3) and p["sfb"].shape == (5, 1, 3)
    assert p["masked_m"].dtype == np.int32 and p["masked_m"].shape == (5,)
    assert (p["masked_m"] >= 0).all() and (p["masked_m"] <= 256).all()
    q = inputs.masked_fp8_problem(5, 256, 96, 384, seed=3)
    assert np.array_equal(p["masked_m"], q["masked_m"]) and np.array_equal(p["A"], q["A"])
    with pytest.raises(ValueError):
        inputs.masked_fp8_problem(2, 128, 64, 128, seed=1, counts=[0, 129])


def test_normal_matrix_is_seeded_and_rounds_to_bf16():
    x = inputs.normal_matrix(300, 256, seed=9)
    assert x.dtype == np.float32 and np.array_equal(x, inputs.normal_matrix(300, 256, seed=9))
    assert not np.array_equal(x, inputs.normal_matrix(300, 256, seed=10))
    bits = inputs.normal_matrix(300, 256, seed=9, bf16=True)
    assert bits.dtype == np.uint16 and np.array_equal(bits, inputs.bf16_operand(x))
