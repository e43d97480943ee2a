"""GPU parity over the whole UE8M0 range: the scale path of every GEMM kind against the oracle.

Block scaling exists so that one tensor can span many binades ("DeepGEMM-Ascend cobre
quantas operações no Ascend 950?", section "Fatores de escala FP8 e o formato UE8M0 no
Ascend": a power-of-two factor per block, and a packing error that shows only as wrong
numbers).  These tests put scale bytes far from the bias 127, down to 1 and up to 254, and
mix magnitudes inside one dot product, while keeping every output inside the bf16 range.

Where each output (m, n) carries a known power-of-two magnitude 2^c[m,n], both the GPU
result and the oracle's fp64 value are divided by it before the stated GEMM tolerance is
applied (dividing by a power of two is exact), so the check is as strict for outputs near
2^-60 as for outputs near 2^60.

Per-row B scales (sfb_gran_n = 1) in the contiguous and masked grouped layouts are also
checked here.
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

    assert ops.device_status() == 0
    return ops


def _status_ok(ops):
    st = ops.device_status()
    assert st == 0, f"device status {st}"


def _finite_e4m3_codes(rng, shape):
    """E4M3 codes of magnitude 2^-4 .. 2^4 (exponent fields 3 .. 11), every sign and mantissa,
    with subnormals and zeros mixed in.  Products then stay within 2^+-8, so the fp32 partial
    sums of a dot product stay small next to the outputs' own size, as for quantised data,
    whatever the (power-of-two) scales are; the scale bytes carry the dynamic range."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << 7
    exp = rng.integers(3, 12, size=shape, dtype=np.uint8)
    exp = np.where(rng.random(shape) < 0.05, 0, exp).astype(np.uint8)  # subnormals and zeros
    man = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return (sign | (exp << 3) | man).astype(np.uint8)


def _range_bytes(rng, rows_a, rows_b, kb, spread=30):
    """UE8M0 bytes spanning the range with a known product per output.

    ea[m, j] = base[j] + da[m] and eb[r, j] = 254 - base[j] + db[r], so the scale of every
    K block of output (m, n) is 2^(ea + eb - 254) = 2^(da[m] + db[r(n)]): the same for all
    blocks of one dot product, while the bytes themselves sweep base[j] over [31, 223]
    (and reach 1 and 254 at the ends of da, db).
    """
    base = np.linspace(spread + 1, 253 - spread, kb).round().astype(np.int64)
    rng.shuffle(base)
    da = rng.integers(-spread, spread + 1, size=rows_a)
    db = rng.integers(-spread, spread + 1, size=rows_b)
    ea = base[None, :] + da[:, None]
    eb = 254 - base[None, :] + db[:, None]
    assert ea.min() >= 1 and ea.max() <= 254 and eb.min() >= 1 and eb.max() <= 254
    return ea.astype(np.uint8), eb.astype(np.uint8), da, db


def _normalised(got, ref, da, db_per_col):
    """got / 2^c and ref / 2^c for c[m, n] = da[m] + db[n] (exact power-of-two division)."""
    c = da[:, None] + db_per_col[None, :]
    s = np.ldexp(1.0, -c)
    return got * s, ref * s


def _out(m, n):
    ldd = (n + 7) // 8 * 8
    return torch.empty((m, ldd), dtype=torch.bfloat16, device="cuda")[:, :n]


# (M, N, K, sfb_gran_n): pair tiles, ragged edges, the transposed small-M path, a split tail
FP8_SHAPES = [(256, 448, 1024, 128), (300, 200, 1024, 1), (96, 1000, 2048, 128), (40, 520, 1024, 1),
              (256, 1024, 4096, 128)]


@pytest.mark.parametrize("m,n,k,gran", FP8_SHAPES)
def test_fp8_scale_bytes_full_range(ops, orc, m, n, k, gran):
    rng = np.random.default_rng(m * 7 + n + gran)
    kb = k // 128
    A = _finite_e4m3_codes(rng, (m, k))
    B = _finite_e4m3_codes(rng, (n, k))
    mn_b = -(-n // gran)
    sfa, sfb, da, db = _range_bytes(rng, m, mn_b, kb)
    D = _out(m, n)
    ops.gemm_fp8_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), D, sfb_gran_n=gran)
    _status_ok(ops)
    ref = orc.gemm_fp8(A, sfa, B, sfb, gran_n=gran)
    got = bf16_to_f64(D)
    assert np.isfinite(got).all()
    g, r = _normalised(got, ref, da, np.repeat(db, gran)[:n])
    check_gemm(g, r, f"fp8 full-range bytes {m}x{n}x{k} gran {gran} plan {ops.gemm_plan('fp8', m, n, k)}")


@pytest.mark.parametrize("m,n,k,gran", [(256, 448, 1024, 128), (64, 700, 1024, 1)])
def test_fp8_extreme_bytes_in_one_dot_product(ops, orc, m, n, k, gran):
    # block 0 of every dot product at A byte 1 / B byte 253, block 1 at A byte 254 / B byte 1,
    # the others near the bias: all products of the same order, so the extreme bytes decide
    # the result
    rng = np.random.default_rng(m + n)
    kb = k // 128
    A = _finite_e4m3_codes(rng, (m, k))
    B = _finite_e4m3_codes(rng, (n, k))
    mn_b = -(-n // gran)
    sfa = rng.integers(125, 130, size=(m, kb)).astype(np.uint8)
    sfb = (254 - sfa.astype(np.int64).mean(axis=0, dtype=np.float64).round()).astype(np.uint8)
    sfb = np.broadcast_to(sfb, (mn_b, kb)).copy()
    sfa[:, 0], sfb[:, 0] = 1, 253
    sfa[:, 1], sfb[:, 1] = 254, 1
    D = _out(m, n)
    ops.gemm_fp8_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), D, sfb_gran_n=gran)
    _status_ok(ops)
    ref = orc.gemm_fp8(A, sfa, B, sfb, gran_n=gran)
    # the extreme blocks matter: dropping either one changes the reference a lot
    for j in (0, 1):
        A_x = A.copy()
        A_x[:, 128 * j:128 * (j + 1)] = 0
        assert np.linalg.norm(orc.gemm_fp8(A_x, sfa, B, sfb, gran_n=gran) - ref) > 0.1 * np.linalg.norm(ref)
    check_gemm(bf16_to_f64(D), ref, f"fp8 extreme bytes {m}x{n}x{k}")


def _spread_rows(x, rng, lo=-50, hi=50, block=1):
    """Multiply each block of `block` rows by its own power of two 2^U[lo, hi)."""
    nb = -(-x.shape[0] // block)
    r = rng.integers(lo, hi, size=nb)
    x *= np.repeat(np.ldexp(np.float32(1.0), r).astype(np.float32), block)[: x.shape[0], None]
    return np.repeat(r, block)[: x.shape[0]]


@pytest.mark.parametrize("m,n,k,gran", [(256, 512, 1024, 128), (200, 300, 2048, 1), (64, 1024, 1024, 128)])
def test_fp8_quantised_spread_operands(ops, orc, m, n, k, gran):
    # fp32 operands whose rows (A) and 128-row blocks or rows (B) sit 2^-50 .. 2^49 apart,
    # quantised on the GPU (codes and packed words bit-exact against the oracle's), then
    # multiplied: scale bytes from about 70 to 180 in one GEMM
    rng = np.random.default_rng(k + gran)
    xa = inputs.normal_matrix(m, k, seed=m)
    xb = inputs.normal_matrix(n, k, seed=n + 1)
    ra = _spread_rows(xa, rng)
    rb = _spread_rows(xb, rng, block=gran)
    qa, sa = ops.quantize_fp8(to_dev(xa), 1)
    qb, sb = ops.quantize_fp8(to_dev(xb), gran)
    ca, ea = orc.quantize_fp8(xa, 1)
    cb, eb = orc.quantize_fp8(xb, gran)
    assert np.array_equal(qa.cpu().numpy(), ca) and np.array_equal(qb.cpu().numpy(), cb)
    assert np.array_equal(sa.cpu().numpy(), orc.sf_pack(ea, ld_out=sa.shape[1]))
    assert np.array_equal(sb.cpu().numpy(), orc.sf_pack(eb, ld_out=sb.shape[1]))
    assert min(int(ea.min()), int(eb.min())) < 100 and max(int(ea.max()), int(eb.max())) > 150
    D = _out(m, n)
    ops.gemm_fp8_nt(qa, sa, qb, sb, D, sfb_gran_n=gran)
    _status_ok(ops)
    ref = orc.gemm_fp8(ca, ea, cb, eb, gran_n=gran)
    g, r = _normalised(bf16_to_f64(D), ref, ra, rb)
    check_gemm(g, r, f"fp8 quantised spread {m}x{n}x{k} gran {gran}")


@pytest.mark.parametrize("m,n,k", [(256, 448, 1024), (130, 250, 512), (48, 704, 1024), (256, 512, 8192)])
def test_fp4_scale_bytes_full_range(ops, orc, m, n, k):
    rng = np.random.default_rng(m + n + k)
    kb = k // 32
    A = rng.integers(0, 256, size=(m, k // 2), dtype=np.uint8)
    B = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    sfa, sfb, da, db = _range_bytes(rng, m, n, kb)
    D = _out(m, n)
    ops.gemm_fp4_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), D)
    _status_ok(ops)
    ref = orc.gemm_fp4(A, sfa, B, sfb)
    got = bf16_to_f64(D)
    assert np.isfinite(got).all()
    g, r = _normalised(got, ref, da, db)
    check_gemm(g, r, f"fp4 full-range bytes {m}x{n}x{k} plan {ops.gemm_plan('fp4', m, n, k)}")


def test_fp4_extreme_bytes_in_one_dot_product(ops, orc):
    m, n, k = 256, 448, 512
    rng = np.random.default_rng(4)
    kb = k // 32
    A = rng.integers(0, 256, size=(m, k // 2), dtype=np.uint8)
    B = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    sfa = np.full((m, kb), 127, np.uint8)
    sfb = np.full((n, kb), 127, np.uint8)
    sfa[:, 0], sfb[:, 0] = 1, 253
    sfa[:, 5], sfb[:, 5] = 254, 1
    sfa[:, 9], sfb[:, 9] = 200, 54
    D = _out(m, n)
    ops.gemm_fp4_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), D)
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), orc.gemm_fp4(A, sfa, B, sfb), "fp4 extreme bytes")


# ------------------------------------------------------------------ per-row B scales, grouped


@pytest.mark.parametrize("counts,n,k", [([100, 0, 150, 50], 448, 512), ([128, 256, 1, 127, 300], 296, 384)])
def test_grouped_per_row_b_scales(ops, orc, counts, n, k):
    p = inputs.grouped_fp8_problem(len(counts), sum(counts), n, k, seed=11 + len(counts), counts=counts,
                                   b_block_rows=1)
    assert p["sfb"].shape == (len(counts), n, k // 128)
    D = ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]),
                                             to_dev(p["m_indices"]), sfb_gran_n=1)
    _status_ok(ops)
    got = bf16_to_f64(D)
    ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"], gran_n=1)
    check_gemm(got, ref, "grouped, per-row B scales")
    assert np.all(got[p["m_indices"] < 0] == 0.0)


def test_grouped_per_row_b_scales_wide_range(ops, orc):
    # per-row B bytes across the range, A rows' bytes paired with them per K block
    counts = [200, 56, 300]
    n, k = 256, 1024
    p = inputs.grouped_fp8_problem(3, sum(counts), n, k, seed=5, counts=counts, b_block_rows=1)
    rng = np.random.default_rng(6)
    m = p["M"]
    sfa, sfb_e, da, db = _range_bytes(rng, m, 3 * n, k // 128)
    sfb = sfb_e.reshape(3, n, k // 128)
    D = ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"]), to_dev(sfa), to_dev(p["B"]), to_dev(sfb),
                                             to_dev(p["m_indices"]), sfb_gran_n=1)
    _status_ok(ops)
    idx = p["m_indices"]
    valid = idx >= 0
    ref = orc.gemm_grouped_fp8(p["A"], sfa, p["B"], sfb, idx, gran_n=1)
    got = bf16_to_f64(D)
    assert np.all(got[~valid] == 0.0)
    # output (m, n) of expert g carries 2^(da[m] + db[g*n + n'])
    c = da[valid][:, None] + db.reshape(3, n)[idx[valid]]
    s = np.ldexp(1.0, -c)
    check_gemm(got[valid] * s, ref[valid] * s, "grouped per-row B, full-range bytes")


@pytest.mark.parametrize("counts,n,k", [([0, 256, 37, 129], 448, 512), ([1, 128, 255, 64, 0, 200], 1000, 1024)])
def test_masked_per_row_b_scales(ops, orc, counts, n, k):
    p = inputs.masked_fp8_problem(len(counts), 256, n, k, seed=3 + len(counts), counts=counts, b_block_rows=1)
    g, max_m = p["G"], p["max_m"]
    sentinel = 0x3C5A
    D = torch.full((g, max_m, n), 0, dtype=torch.int16, device="cuda").fill_(sentinel).view(torch.bfloat16)
    ops.m_grouped_gemm_fp8_nt_masked(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]),
                                     to_dev(p["masked_m"]), D, sfb_gran_n=1)
    _status_ok(ops)
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16).reshape(g * max_m, n)
    valid = np.concatenate([np.arange(max_m) < c for c in p["masked_m"]])
    assert (raw[~valid] == sentinel).all(), "rows past masked_m were written"
    ref = orc.gemm_masked_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["masked_m"], gran_n=1)
    check_gemm(bf16_to_f64(D).reshape(g * max_m, n)[valid], ref[valid], f"masked per-row B {counts}")


def test_masked_equals_contiguous_per_row_b_scales(ops):
    counts = [1, 128, 77, 5]
    p = inputs.masked_fp8_problem(4, 128, 448, 1024, seed=19, counts=counts, b_block_rows=1)
    D = torch.empty((4, 128, 448), dtype=torch.bfloat16, device="cuda")
    ops.m_grouped_gemm_fp8_nt_masked(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]),
                                     to_dev(p["masked_m"]), D, sfb_gran_n=1)
    idx = np.concatenate([np.where(np.arange(128) < c, g, -1) for g, c in enumerate(counts)]).astype(np.int32)
    Dc = ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"].reshape(512, 1024)), to_dev(p["sfa"]), to_dev(p["B"]),
                                              to_dev(p["sfb"]), to_dev(idx), sfb_gran_n=1)
    _status_ok(ops)
    valid = torch.from_numpy(idx >= 0).cuda()
    assert torch.equal(D.reshape(512, 448)[valid].view(torch.int16), Dc[valid].view(torch.int16))
