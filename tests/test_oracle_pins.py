"""Pins for the CPU oracle: each checks it against something other than itself.

* decode tables against ml_dtypes (an independent implementation of the OCP
  E4M3 / E2M1 / E8M0 formats) and against values fixed by the bit-field
  definitions;
* the GEMMs against exact rational brute force (fractions.Fraction, decoding by
  ml_dtypes) on tiny shapes, and against closed forms (identity, all-ones,
  single non-unit scale);
* the SF packing against a hand-worked example and the pack/unpack round trip;
* the bf16 rounding against brute-force nearest-even over all bf16 values;
* the quantiser against ml_dtypes' E4M3 rounding, the defining inequality of the
  block exponent, hand-worked blocks (ties, subnormals, signed zeros, the clamp)
  and the input generator's independent numpy quantiser.
"""

from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest


def _all_e4m3():
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def _all_e2m1():
    return np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _all_e8m0():
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)


# ---------------------------------------------------------------- decode tables

def test_decode_tables_match_ml_dtypes(orc):
    e4, e2, u8 = orc.tables()
    ref4, ref2, ref8 = _all_e4m3(), _all_e2m1(), _all_e8m0()
    assert np.array_equal(np.isnan(e4), np.isnan(ref4))
    assert np.array_equal(e4[~np.isnan(e4)], ref4[~np.isnan(ref4)])
    assert np.array_equal(e2, ref2)
    assert np.array_equal(np.isnan(u8), np.isnan(ref8))
    assert np.array_equal(u8[~np.isnan(u8)], ref8[~np.isnan(ref8)])


def test_decode_spot_values(orc):
    e4, e2, u8 = orc.tables()
    # E4M3FN: sign|eeee|mmm, bias 7
    assert e4[0x38] == 1.0 and e4[0xB8] == -1.0
    assert e4[0x7E] == 448.0 and e4[0xFE] == -448.0  # largest finite
    assert e4[0x08] == 2.0 ** -6  # smallest normal
    assert e4[0x01] == 2.0 ** -9  # smallest subnormal
    assert e4[0x07] == 7 * 2.0 ** -9
    assert e4[0x00] == 0.0 and np.signbit(e4[0x80])
    assert np.isnan(e4[0x7F]) and np.isnan(e4[0xFF])
    assert int(np.isnan(e4).sum()) == 2  # no infinities, only S.1111.111 is NaN
    # E2M1 magnitudes
    assert list(e2[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(e2[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    # UE8M0
    assert u8[127] == 1.0 and u8[128] == 2.0 and u8[126] == 0.5
    assert u8[0] == 2.0 ** -127 and u8[254] == 2.0 ** 127 and np.isnan(u8[255])


# ------------------------------------------------------------------ SF packing

def test_sf_pack_hand_example(orc):
    # two rows, three K blocks (odd: the last word's high byte is empty), ld 4
    e = np.array([[127, 128, 5], [0, 254, 1]], np.uint8)
    w = orc.sf_pack(e, ld_out=4).view(np.uint16)
    assert w.shape == (2, 4)
    assert list(w[0]) == [0x807F, 0xFE00, 0, 0]  # low byte = even block, high byte = odd block
    assert list(w[1]) == [0x0005, 0x0001, 0, 0]


@pytest.mark.parametrize("mn,kb,pad", [(1, 2, 7), (37, 8, 3), (128, 56, 0), (300, 5, 4), (8, 1, 0)])
def test_sf_pack_roundtrip(orc, mn, kb, pad):
    rng = np.random.default_rng(mn * 100 + kb)
    e = rng.integers(0, 255, size=(mn, kb), dtype=np.uint8)
    w = orc.sf_pack(e, ld_out=mn + pad)
    assert w.shape == ((kb + 1) // 2, mn + pad) and w.dtype == np.int16
    assert np.array_equal(orc.sf_unpack(w, mn, kb), e)
    u = w.view(np.uint16)
    assert not u[:, mn:].any()  # padding columns are zero
    if kb % 2:
        assert not (u[-1, :mn] >> 8).any()
    # MN-major: word j of row r sits at flat index j*ld + r
    flat = u.reshape(-1)
    j, r = (kb - 1) // 2, mn - 1
    hi = int(e[r, 2 * j + 1]) if 2 * j + 1 < kb else 0
    assert int(flat[j * (mn + pad) + r]) == int(e[r, 2 * j]) | (hi << 8)


def test_fp32_scale_conversion(orc):
    good = np.array([1.0, 2.0, 0.5, 2.0 ** -126, 2.0 ** 127, 2.0 ** -7], np.float32)
    assert list(orc.fp32_scales_to_ue8m0(good)) == [127, 128, 126, 1, 254, 120]
    for bad in (3.0, 0.0, -1.0, np.inf, np.nan, 2.0 ** -127, 1.5):
        with pytest.raises(ValueError):
            orc.fp32_scales_to_ue8m0(np.array([bad], np.float32))


# ------------------------------------------------------------------ bf16 round

def _bf16_brute(x):
    allv = np.arange(0x7F80, dtype=np.uint32)  # non-negative finite bf16
    vals = (allv << 16).view(np.float32).astype(np.float64)
    a = abs(x)
    i = np.searchsorted(vals, a)
    cands = [c for c in (i - 1, i) if 0 <= c < len(vals)]
    best = min(cands, key=lambda c: (abs(vals[c] - a), c & 1))
    bits = int(allv[best])
    return bits | (0x8000 if x < 0 else 0)


def test_bf16_round_brute(orc):
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(300) * 10.0 ** rng.integers(-8, 8, 300),
                        # exact ties: 1 + 2^-8 (tie, even -> 1.0), 1 + 3*2^-8 (tie, even -> 1+2^-6)
                        np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.0 ** -130, 0.0])])
    got = orc.bf16_round(x)
    for xi, gi in zip(x, got):
        assert int(gi) == _bf16_brute(xi), xi
    assert int(got[-5]) == 0x3F80 and int(got[-4]) == 0x3F82


# --------------------------------------------------------------- GEMM brute force

def _frac(v):
    return Fraction(float(v))


def _brute_fp8(A, sfa, B, sfb, gran_n):
    a = A.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    b = B.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    m, k = A.shape
    n = B.shape[0]
    out = np.empty((m, n), object)
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                sa = Fraction(2) ** (int(sfa[i, kk // 128]) - 127)
                sb = Fraction(2) ** (int(sfb[j // gran_n, kk // 128]) - 127)
                acc += _frac(a[i, kk]) * _frac(b[j, kk]) * sa * sb
            out[i, j] = acc
    return out


def _finite_e4m3_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7F) == 0x7F, c & 0xFE, c).astype(np.uint8)  # drop the NaN codes


@pytest.mark.parametrize("gran_n", [1, 128, 2])
def test_fp8_gemm_exact_vs_fraction(orc, gran_n):
    rng = np.random.default_rng(11 + gran_n)
    m, n, k = 3, 4, 256
    A = _finite_e4m3_codes(rng, (m, k))
    B = _finite_e4m3_codes(rng, (n, k))
    sfa = rng.integers(118, 137, size=(m, k // 128), dtype=np.uint8)
    sfb = rng.integers(118, 137, size=(-(-n // gran_n), k // 128), dtype=np.uint8)
    D = orc.gemm_fp8(A, sfa, B, sfb, gran_n=gran_n)
    ref = _brute_fp8(A, sfa, B, sfb, gran_n)
    for i in range(m):
        for j in range(n):
            assert Fraction(D[i, j]) == ref[i, j]  # exact: fp64 holds the whole sum


def test_fp8_all_code_pairs(orc):
    # every finite code of A against every finite code of B, one product per output
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    A = np.zeros((codes.size, 128), np.uint8)
    A[:, 0] = codes
    B = np.zeros((codes.size, 128), np.uint8)
    B[:, 0] = codes
    sfa = np.full((codes.size, 1), 127, np.uint8)
    sfb = np.full((codes.size, 1), 127, np.uint8)
    D = orc.gemm_fp8(A, sfa, B, sfb, gran_n=1)
    v = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(D, np.outer(v, v))


def test_fp4_gemm_exact_vs_fraction(orc):
    rng = np.random.default_rng(3)
    m, n, k = 3, 2, 128
    A = rng.integers(0, 256, size=(m, k // 2), dtype=np.uint8)
    B = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    sfa = rng.integers(120, 135, size=(m, k // 32), dtype=np.uint8)
    sfb = rng.integers(120, 135, size=(n, k // 32), dtype=np.uint8)
    D = orc.gemm_fp4(A, sfa, B, sfb)
    e2 = _all_e2m1()

    def elem(P, r, kk):  # even K index in the low nibble
        return e2[(P[r, kk // 2] >> (4 * (kk % 2))) & 0xF]

    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                s = Fraction(2) ** (int(sfa[i, kk // 32]) + int(sfb[j, kk // 32]) - 254)
                acc += _frac(elem(A, i, kk)) * _frac(elem(B, j, kk)) * s
            assert Fraction(D[i, j]) == acc


def test_fp4_nibble_order(orc):
    # one non-zero value at K index 1 (the high nibble of byte 0)
    A = np.zeros((1, 32), np.uint8)
    A[0, 0] = 0x70  # element 1 = 6.0, element 0 = 0
    B = np.zeros((1, 32), np.uint8)
    B[0, 0] = 0x02  # element 0 = 1.0, element 1 = 0
    sf = np.full((1, 2), 127, np.uint8)
    assert orc.gemm_fp4(A, sf, B, sf)[0, 0] == 0.0
    B[0, 0] = 0x20  # element 1 = 1.0
    assert orc.gemm_fp4(A, sf, B, sf)[0, 0] == 6.0


def test_bf16_gemm_vs_fraction(orc):
    rng = np.random.default_rng(4)
    m, n, k = 2, 3, 64
    A = rng.standard_normal((m, k)).astype(ml_dtypes.bfloat16)
    B = rng.standard_normal((n, k)).astype(ml_dtypes.bfloat16)
    D = orc.gemm_bf16(A.view(np.uint16), B.view(np.uint16))
    for i in range(m):
        for j in range(n):
            ref = sum(_frac(A[i, kk].astype(np.float64)) * _frac(B[j, kk].astype(np.float64)) for kk in range(k))
            assert abs(Fraction(D[i, j]) - ref) <= Fraction(2) ** -40 * (1 + abs(ref))


# ------------------------------------------------------------------ closed forms

def test_identity_fp8(orc):
    # A = I (E4M3 1.0 = 0x38, unit scales): D[m, n] = B[n, m] * sfb scale, exactly
    k = 256
    A = np.zeros((k, k), np.uint8)
    A[np.arange(k), np.arange(k)] = 0x38
    sfa = np.full((k, 2), 127, np.uint8)
    rng = np.random.default_rng(9)
    n = 130
    B = _finite_e4m3_codes(rng, (n, k))
    sfb = rng.integers(120, 134, size=(2, 2), dtype=np.uint8)
    D = orc.gemm_fp8(A, sfa, B, sfb, gran_n=128)
    b = B.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    scale = 2.0 ** (sfb.astype(np.int64) - 127)
    expect = b.T * scale[np.arange(n) // 128][:, np.arange(k) // 128].T
    assert np.array_equal(D, expect)


@pytest.mark.parametrize("a,b", [(0, 0), (3, -5), (-20, 11)])
def test_all_ones_fp8(orc, a, b):
    m, n, k = 5, 7, 512
    A = np.full((m, k), 0x38, np.uint8)
    B = np.full((n, k), 0x38, np.uint8)
    sfa = np.full((m, k // 128), 127 + a, np.uint8)
    sfb = np.full((1, k // 128), 127 + b, np.uint8)
    assert np.all(orc.gemm_fp8(A, sfa, B, sfb) == k * 2.0 ** (a + b))


def test_all_ones_fp4(orc):
    m, n, k = 3, 4, 256
    A = np.full((m, k // 2), 0x22, np.uint8)  # 1.0 in both nibbles
    B = np.full((n, k // 2), 0x22, np.uint8)
    sfa = np.full((m, k // 32), 129, np.uint8)
    sfb = np.full((n, k // 32), 125, np.uint8)
    assert np.all(orc.gemm_fp4(A, sfa, B, sfb) == k * 1.0)


def test_single_scale_localises(orc):
    # one non-unit (row, K-block) scale of A changes exactly that row by that block's share
    rng = np.random.default_rng(21)
    m, n, k = 6, 5, 512
    A = _finite_e4m3_codes(rng, (m, k))
    B = _finite_e4m3_codes(rng, (n, k))
    sfa = np.full((m, k // 128), 127, np.uint8)
    sfb = np.full((1, k // 128), 127, np.uint8)
    D0 = orc.gemm_fp8(A, sfa, B, sfb)
    sfa2 = sfa.copy()
    sfa2[4, 2] = 130
    D1 = orc.gemm_fp8(A, sfa2, B, sfb)
    a = A.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    b = B.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    part = a[4, 256:384] @ b[:, 256:384].T
    changed = np.argwhere(D1 != D0)
    assert set(changed[:, 0]) <= {4}
    assert np.allclose(D1[4] - D0[4], 7.0 * part, rtol=0, atol=1e-9 * np.abs(part).max())


def test_grouped_equals_dense_slices(orc):
    import inputs

    p = inputs.grouped_fp8_problem(4, 300, 256, 256, seed=7, counts=[100, 0, 150, 50])
    D = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"])
    starts = np.concatenate([[0], np.cumsum(((p["counts"] + 127) // 128) * 128)])
    assert p["M"] == 128 + 0 + 256 + 128
    for g in range(4):
        s, c = int(starts[g]), int(p["counts"][g])
        if c == 0:
            continue
        dense = orc.gemm_fp8(p["A"][s:s + c], p["sfa"][s:s + c], p["B"][g], p["sfb"][g])
        assert np.array_equal(D[s:s + c], dense)
    pad = p["m_indices"] < 0
    assert pad.sum() == p["M"] - 300 and np.all(D[pad] == 0.0)
    # rows with expert index -1 are 0 whatever A holds there
    A2 = p["A"].copy()
    A2[pad] = 0x38
    D2 = orc.gemm_grouped_fp8(A2, p["sfa"], p["B"], p["sfb"], p["m_indices"])
    assert np.array_equal(D2, D)
    bad = p["m_indices"].copy()
    bad[0] = 4
    with pytest.raises(ValueError):
        orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], bad)


def test_sampled_equals_full(orc):
    import inputs

    p = inputs.dense_fp8_problem(64, 96, 512, seed=2)
    full = orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"])
    rows, cols = np.array([0, 63, 17]), np.array([95, 0, 40, 41])
    assert np.array_equal(orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], rows=rows, cols=cols),
                          full[np.ix_(rows, cols)])


# ---------------------------------------------------------------- quantiser

def _quant_data(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    # spread the block magnitudes over many binades, including tiny and huge ones
    rs = np.ldexp(np.float32(1.0), rng.integers(-60, 60, size=(rows, 1))).astype(np.float32)
    x = (x * rs).astype(np.float32)
    x[0, :128] = 0.0                      # an all-zero block
    x[1 % rows, 5] = -0.0
    x[-1, -128:] *= np.float32(2.0 ** -100)  # a block below the clamp (e < -126)
    return x


@pytest.mark.parametrize("block_rows,rows", [(1, 37), (128, 300), (128, 128)])
def test_quantize_matches_ml_dtypes_rounding(orc, block_rows, rows):
    x = _quant_data(rows, 384, seed=rows)
    q, e = orc.quantize_fp8(x, block_rows)
    exp = e.astype(np.int32) - 127
    scale = np.repeat(np.repeat(np.ldexp(1.0, -exp), block_rows, axis=0)[:rows], 128, axis=1)
    scaled = (x.astype(np.float64) * scale).astype(np.float32)  # exact: powers of two, no underflow here
    ref = scaled.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(q, ref)


@pytest.mark.parametrize("block_rows", [1, 128])
def test_quantize_exponent_is_the_smallest_that_fits(orc, block_rows):
    x = _quant_data(260, 256, seed=block_rows)
    _, e = orc.quantize_fp8(x, block_rows)
    rb = -(-260 // block_rows)
    pad = np.zeros((rb * block_rows - 260, 256), np.float32)
    amax = np.abs(np.concatenate([x, pad])).astype(np.float64).reshape(rb, block_rows, 2, 128).max(axis=(1, 3))
    ex = e.astype(np.int64) - 127
    free = (amax > 0) & (ex > -126)          # not zero, not clamped
    assert np.all(448.0 * np.ldexp(1.0, ex) >= amax)
    assert np.all(448.0 * np.ldexp(1.0, ex[free] - 1) < amax[free])
    assert np.all(e[amax == 0] == 127)
    assert np.all(e[(amax > 0) & (amax < 448.0 * 2.0 ** -127)] == 1)  # clamped at the UE8M0 floor


def test_quantize_hand_blocks(orc):
    x = np.zeros((4, 128), np.float32)
    # row 0: amax exactly 448 * 2^3 -> e = 3, 448 * 2^3 -> 448 (0x7E); ties in units of 2^3
    x[0, 0] = 448.0 * 8
    x[0, 1] = (1.0 + 1.0 / 16) * 8   # halfway 1 .. 1.125 -> even mantissa 0: 1.0 = 0x38
    x[0, 2] = (1.0 + 3.0 / 16) * 8   # halfway 1.125 .. 1.25 -> even mantissa 2: 1.25 = 0x3A
    x[0, 3] = -(2.0 ** -10) * 8      # halfway 0 .. 2^-9 -> 0, sign kept: 0x80
    x[0, 4] = (3.0 * 2.0 ** -10) * 8  # halfway 2^-9 .. 2^-8 -> even: 2^-8 = 0x02
    x[0, 5] = (15.5 / 8) * 8 * 2.0 ** 7  # 1.9375 * 2^7 * 2^3: halfway 1.875..2 (binade 7) -> 2^8 = 0x78
    # row 1: amax just above 448 -> e = 1, and 448.0 * (1 + 2^-20) / 2 -> 224 (0x76)
    x[1, 0] = 448.0 * (1 + 2.0 ** -20)
    # row 2: all zero, one negative zero -> byte 127, codes 0x00 / 0x80
    x[2, 7] = -0.0
    # row 3: amax 1.0 -> smallest e with 448 * 2^e >= 1 is -8 (448/256 = 1.75)
    x[3, 0] = 1.0
    x[3, 1] = -0.5
    q, e = orc.quantize_fp8(x, 1)
    assert list(e[:, 0]) == [130, 128, 127, 119]
    assert list(q[0, :6]) == [0x7E, 0x38, 0x3A, 0x80, 0x02, 0x78]
    assert q[1, 0] == 0x76
    assert q[2, 7] == 0x80 and not q[2, :7].any() and not q[2, 8:].any()
    # row 3: 1.0 * 2^8 = 256 = 1.0 * 2^8 -> exponent field 15, mantissa 0 = 0x78; -0.5 * 2^8 = -128 -> 0xF0
    assert q[3, 0] == 0x78 and q[3, 1] == 0xF0


def test_quantize_bf16_input_is_its_exact_fp32_value(orc):
    rng = np.random.default_rng(3)
    bits = rng.standard_normal((8, 256)).astype(np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)
    f32 = (bits.astype(np.uint32) << 16).view(np.float32)
    for br in (1, 128):
        qa, ea = orc.quantize_fp8(bits, br)
        qb, eb = orc.quantize_fp8(f32, br)
        assert np.array_equal(qa, qb) and np.array_equal(ea, eb)


def test_quantize_rejects_non_finite(orc):
    x = np.ones((2, 128), np.float32)
    x[1, 3] = np.inf
    with pytest.raises(ValueError):
        orc.quantize_fp8(x, 1)


@pytest.mark.parametrize("block_rows", [1, 128])
def test_quantize_agrees_with_the_input_generator(orc, block_rows):
    import inputs

    x = np.random.default_rng(11).standard_normal((300, 512)).astype(np.float32)
    q, e = orc.quantize_fp8(x, block_rows)
    q2, e2 = inputs.quantize_e4m3_blocks(x, block_rows)
    assert np.array_equal(q, q2) and np.array_equal(e, e2)


# ---------------------------------------------------------------- masked grouped

def test_masked_equals_dense_per_expert(orc):
    import inputs

    p = inputs.masked_fp8_problem(4, 128, 96, 256, seed=5, counts=[0, 128, 37, 1])
    got = orc.gemm_masked_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["masked_m"]).reshape(4, 128, 96)
    for g, c in enumerate(p["masked_m"]):
        if c:
            ref = orc.gemm_fp8(p["A"][g, :c], p["sfa"][g * 128:g * 128 + c], p["B"][g], p["sfb"][g])
            assert np.array_equal(got[g, :c], ref)
        assert np.isnan(got[g, c:]).all()


def test_masked_exact_vs_fraction(orc):
    rng = np.random.default_rng(8)
    G, max_m, n, k = 2, 3, 2, 128
    codes = _all_e4m3()
    ok = np.flatnonzero(~np.isnan(codes)).astype(np.uint8)
    A = rng.choice(ok, size=(G, max_m, k)).astype(np.uint8)
    B = rng.choice(ok, size=(G, n, k)).astype(np.uint8)
    sfa = rng.integers(120, 134, size=(G * max_m, 1)).astype(np.uint8)
    sfb = rng.integers(120, 134, size=(G, 1, 1)).astype(np.uint8)
    mm = np.array([2, 3], np.int32)
    got = orc.gemm_masked_fp8(A, sfa, B, sfb, mm)
    for g in range(G):
        for m in range(max_m):
            for j in range(n):
                v = got[g * max_m + m, j]
                if m >= mm[g]:
                    assert np.isnan(v)
                    continue
                s = sum(Fraction(codes[A[g, m, q]]) * Fraction(codes[B[g, j, q]]) for q in range(k))
                ref = s * Fraction(2) ** (int(sfa[g * max_m + m, 0]) - 127) * Fraction(2) ** (int(sfb[g, 0, 0]) - 127)
                assert Fraction(v) == ref


def test_masked_rejects_counts_out_of_range(orc):
    import inputs

    p = inputs.masked_fp8_problem(2, 128, 64, 128, seed=1, counts=[3, 4])
    with pytest.raises(ValueError):
        orc.gemm_masked_fp8(p["A"], p["sfa"], p["B"], p["sfb"], np.array([3, 129], np.int32))
