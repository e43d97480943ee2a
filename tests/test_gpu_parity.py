"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Inputs come from the seeded generators in ``inputs``; the GPU path packs the scale
factors with its own transform kernel, the oracle reads the unpacked UE8M0 bytes.
Bit-exact where the result is unique (scale transform, identity closed form, G=1
grouped = dense); the stated GEMM tolerance (tests/parity.py) elsewhere.
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



# ------------------------------------------------------------------ SF transform

@pytest.mark.parametrize("mn,kb,ld_pad", [(256, 8, 0), (37, 5, 3), (1, 1, 7), (4096, 128, 0), (300, 130, 12)])
def test_transform_bit_exact_u8(ops, orc, mn, kb, ld_pad):
    rng = np.random.default_rng(mn + kb)
    e = rng.integers(0, 255, size=(mn, kb), dtype=np.uint8)
    ld = (mn + 7) // 8 * 8 + 8 * ld_pad
    got = ops.transform_sf_ue8m0(to_dev(e), ld_out=ld)
    _status_ok(ops)
    assert np.array_equal(got.cpu().numpy(), orc.sf_pack(e, ld_out=ld))


@pytest.mark.parametrize("mn,kb", [(36864, 56), (7168, 512), (129, 3)])
def test_transform_bit_exact_fp32(ops, orc, mn, kb):
    rng = np.random.default_rng(kb)
    e = rng.integers(1, 255, size=(mn, kb), dtype=np.uint8)
    s = np.ldexp(np.float32(1.0), e.astype(np.int32) - 127).astype(np.float32)
    got = ops.transform_sf_ue8m0(to_dev(s))
    _status_ok(ops)
    ld = (mn + 7) // 8 * 8
    assert np.array_equal(got.cpu().numpy(), orc.sf_pack(orc.fp32_scales_to_ue8m0(s), ld_out=ld))


# The transform loads along K as wide as the input's row stride allows (16, 8, 4 or 1 bytes):
# every width, a vector cut short at the end of a row, several K tiles and a padded ld_out.
@pytest.mark.parametrize("kind,mn,kb,ld_in", [("u8", 300, 64, 64), ("u8", 257, 56, 56), ("u8", 130, 40, 48),
                                              ("u8", 99, 20, 20), ("u8", 64, 130, 130), ("fp32", 200, 6, 8),
                                              ("fp32", 333, 5, 6), ("fp32", 77, 3, 3), ("fp32", 1000, 150, 152)])
def test_transform_vector_widths(ops, orc, kind, mn, kb, ld_in):
    rng = np.random.default_rng(mn * kb)
    e = rng.integers(1, 255, size=(mn, kb), dtype=np.uint8)
    full = np.zeros((mn, ld_in), np.uint8 if kind == "u8" else np.float32)
    if kind == "u8":
        full[:, :kb] = e
    else:
        full[:, :kb] = np.ldexp(np.float32(1.0), e.astype(np.int32) - 127)
    src = to_dev(full)[:, :kb]
    ld_out = (mn + 7) // 8 * 8 + 8
    got = ops.transform_sf_ue8m0(src, ld_out=ld_out)
    _status_ok(ops)
    assert np.array_equal(got.cpu().numpy(), orc.sf_pack(e, ld_out=ld_out))


# Two conversions in one launch (a GEMM's A and B scales): the same bytes as two single calls
# and as the oracle's packing, whichever tensor is larger, with different load widths and padded
# outputs.
@pytest.mark.parametrize("kind,mn_a,mn_b,kb,ld_in_a,ld_in_b", [("u8", 4096, 56, 128, 128, 128),
                                                               ("u8", 37, 300, 5, 5, 8),
                                                               ("fp32", 4096, 7168, 512, 512, 512),
                                                               ("fp32", 129, 7, 3, 3, 4), ("u8", 1, 1, 1, 1, 1)])
def test_transform_pair_matches_single_calls_and_oracle(ops, orc, kind, mn_a, mn_b, kb, ld_in_a, ld_in_b):
    rng = np.random.default_rng(mn_a + 3 * mn_b + kb)
    srcs, es = [], []
    for mn, ld_in in ((mn_a, ld_in_a), (mn_b, ld_in_b)):
        e = rng.integers(1, 255, size=(mn, kb), dtype=np.uint8)
        full = np.zeros((mn, ld_in), np.uint8 if kind == "u8" else np.float32)
        full[:, :kb] = e if kind == "u8" else np.ldexp(np.float32(1.0), e.astype(np.int32) - 127)
        srcs.append(to_dev(full)[:, :kb])
        es.append(e)
    lds = [(mn_a + 7) // 8 * 8 + 8, (mn_b + 7) // 8 * 8 + 16]
    outs = [torch.full(((kb + 1) // 2, ld), -1, dtype=torch.int16, device="cuda") for ld in lds]
    ops.transform_sf_ue8m0_pair(srcs[0], srcs[1], out_a=outs[0], out_b=outs[1])
    _status_ok(ops)
    for src, e, out, ld in zip(srcs, es, outs, lds):
        assert np.array_equal(out.cpu().numpy(), orc.sf_pack(e, ld_out=ld))
        assert torch.equal(out, ops.transform_sf_ue8m0(src, ld_out=ld))


def test_transform_pair_flags_nan_byte_in_either(ops, orc):
    a = np.full((300, 6), 127, np.uint8)
    b = np.full((20, 6), 127, np.uint8)
    b[19, 0] = 0xFF
    out_a, out_b = ops.transform_sf_ue8m0_pair(to_dev(a), to_dev(b))
    assert ops.device_status() == -7
    _status_ok(ops)  # cleared
    assert np.array_equal(out_b.cpu().numpy(), orc.sf_pack(b, ld_out=out_b.shape[1]))
    assert np.array_equal(out_a.cpu().numpy(), orc.sf_pack(a, ld_out=out_a.shape[1]))


# A stack of same-shaped tensors in one launch (per-expert B scales): each tensor the bytes a
# single call and the oracle give, with gaps between the input rows and between the tensors on
# both sides, and a batch of one.
@pytest.mark.parametrize("kind,g,mn,kb,row_pad,gap_in,ld_pad,gap_out", [("u8", 32, 32, 56, 0, 0, 0, 0),
                                                                        ("u8", 5, 300, 7, 1, 13, 8, 16),
                                                                        ("fp32", 3, 129, 5, 3, 4, 0, 8),
                                                                        ("fp32", 1, 40, 512, 0, 0, 16, 0)])
def test_transform_batched_matches_single_calls_and_oracle(ops, orc, kind, g, mn, kb, row_pad, gap_in, ld_pad,
                                                           gap_out):
    rng = np.random.default_rng(g * mn + kb)
    e = rng.integers(1, 255, size=(g, mn, kb), dtype=np.uint8)
    ld_in = kb + row_pad
    flat = np.zeros(g * (mn * ld_in + gap_in), np.uint8 if kind == "u8" else np.float32)
    full = np.lib.stride_tricks.as_strided(flat, shape=(g, mn, ld_in),
                                           strides=(flat.itemsize * (mn * ld_in + gap_in), flat.itemsize * ld_in,
                                                    flat.itemsize))
    full[:, :, :kb] = e if kind == "u8" else np.ldexp(np.float32(1.0), e.astype(np.int32) - 127)
    dflat = to_dev(flat)
    src = dflat.as_strided((g, mn, kb), (mn * ld_in + gap_in, ld_in, 1))
    words, ld = (kb + 1) // 2, (mn + 7) // 8 * 8 + ld_pad
    oflat = torch.full((g * (words * ld + gap_out),), -1, dtype=torch.int16, device="cuda")
    out = oflat.as_strided((g, words, ld), (words * ld + gap_out, ld, 1))
    ops.transform_sf_ue8m0_batched(src, out=out)
    _status_ok(ops)
    got = out.cpu().numpy()
    for z in range(g):
        assert np.array_equal(got[z], orc.sf_pack(e[z], ld_out=ld)), z
        assert torch.equal(out[z], ops.transform_sf_ue8m0(src[z], ld_out=ld)), z
    if gap_out:  # the gaps between output tensors are not written
        gaps = oflat.view(g, -1)[:, words * ld:].cpu().numpy()
        assert (gaps == -1).all()


def test_transform_batched_flags_nan_byte(ops):
    e = np.full((4, 20, 6), 127, np.uint8)
    e[2, 19, 5] = 0xFF
    ops.transform_sf_ue8m0_batched(to_dev(e))
    assert ops.device_status() == -7
    _status_ok(ops)  # cleared


def test_transform_flags_bad_scale(ops):
    s = np.ones((16, 4), np.float32)
    s[3, 2] = 3.0
    ops.transform_sf_ue8m0(to_dev(s))
    assert ops.device_status() == -7
    _status_ok(ops)  # cleared


def test_transform_flags_nan_byte(ops, orc):
    # UE8M0 0xFF is NaN: the uint8 path latches the check too, and still packs the byte
    e = np.full((40, 6), 127, np.uint8)
    e[21, 5] = 0xFF
    got = ops.transform_sf_ue8m0(to_dev(e))
    assert ops.device_status() == -7
    _status_ok(ops)  # cleared
    assert np.array_equal(got.cpu().numpy(), orc.sf_pack(e, ld_out=got.shape[1]))


def test_reuse_or_convert(ops):
    e = to_dev(np.full((256, 8), 127, np.uint8))
    packed = ops.packed_sf(e, 256, 8)
    assert packed.dtype == torch.int16 and tuple(packed.shape) == (4, 256)
    assert ops.packed_sf(packed, 256, 8) is packed  # already packed: reused, not converted


# ------------------------------------------------------------------ FP8

def _fp8_case(ops, orc, m, n, k, seed, gran, fp32_scales=False):
    p = inputs.dense_fp8_problem(m, n, k, seed=seed, b_block_rows=gran)
    sfa, sfb = p["sfa"], p["sfb"]
    if fp32_scales:
        sfa = np.ldexp(np.float32(1), sfa.astype(np.int32) - 127).astype(np.float32)
        sfb = np.ldexp(np.float32(1), sfb.astype(np.int32) - 127).astype(np.float32)
    ldd = (n + 7) // 8 * 8  # rows of D must start 16-byte aligned
    D = torch.empty((m, ldd), dtype=torch.bfloat16, device="cuda")[:, :n]
    ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(sfa), to_dev(p["B"]), to_dev(sfb), D, sfb_gran_n=gran)
    _status_ok(ops)
    ref = orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=gran)
    return check_gemm(bf16_to_f64(D), ref, f"fp8 {m}x{n}x{k} gran {gran}")


def test_fp8_config0(ops, orc):
    # 256 x 512 x 1024, 1x128 A scales, 128x128 B scales, scales packed on the GPU
    _fp8_case(ops, orc, 256, 512, 1024, seed=0, gran=128)


@pytest.mark.parametrize("m,n,k,gran", [(200, 300, 384, 128), (130, 232, 256, 1), (1, 1024, 128, 128),
                                        (300, 8, 256, 1), (129, 449, 640, 1), (384, 672, 2048, 128)])
def test_fp8_ragged(ops, orc, m, n, k, gran):
    _fp8_case(ops, orc, m, n, k, seed=m + n, gran=gran)


def test_fp8_fp32_scale_inputs(ops, orc):
    _fp8_case(ops, orc, 256, 448, 512, seed=3, gran=128, fp32_scales=True)


def test_fp8_identity_bit_exact(ops, orc):
    # A = I (E4M3 1.0 = 0x38) with unit scales: D = B^T * scale exactly, representable in bf16
    k = 256
    A = np.zeros((k, k), np.uint8)
    A[np.arange(k), np.arange(k)] = 0x38
    sfa = np.full((k, 2), 127, np.uint8)
    rng = np.random.default_rng(9)
    n = 448
    B = rng.integers(0, 256, size=(n, k), dtype=np.uint8)
    B = np.where((B & 0x7F) == 0x7F, B & 0xFE, B).astype(np.uint8)
    sfb = rng.integers(118, 136, size=(4, 2), dtype=np.uint8)
    D = ops.gemm_fp8_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), sfb_gran_n=128)
    _status_ok(ops)
    ref = orc.gemm_fp8(A, sfa, B, sfb, gran_n=128)
    assert np.array_equal(D.view(torch.int16).cpu().numpy().view(np.uint16), orc.bf16_round(ref))


@pytest.mark.parametrize("m,n,gran", [(1, 8, 128), (1, 1, 1), (3, 17, 128)])
def test_fp8_degenerate_shapes_bit_exact(ops, orc, m, n, gran):
    # a handful of outputs: each row of A picks one K column (E4M3 1.0), so every output is
    # one decoded B value times its scales, exactly representable in bf16
    k = 256
    rng = np.random.default_rng(m * 31 + n)
    A = np.zeros((m, k), np.uint8)
    A[np.arange(m), rng.integers(0, k, m)] = 0x38
    B = rng.integers(0, 256, size=(n, k), dtype=np.uint8)
    B = np.where((B & 0x7F) == 0x7F, B & 0xFE, B).astype(np.uint8)
    sfa = rng.integers(120, 134, size=(m, 2), dtype=np.uint8)
    sfb = rng.integers(120, 134, size=(-(-n // gran), 2), dtype=np.uint8)
    ldd = (n + 7) // 8 * 8
    D = torch.zeros((m, ldd), dtype=torch.bfloat16, device="cuda")
    ops.gemm_fp8_nt(to_dev(A), to_dev(sfa), to_dev(B), to_dev(sfb), D[:, :n], sfb_gran_n=gran)
    _status_ok(ops)
    got = D.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got[:, :n], orc.bf16_round(orc.gemm_fp8(A, sfa, B, sfb, gran_n=gran)))
    assert not got[:, n:].any()  # nothing written past column N


def test_fp8_single_scale_localises(ops, orc):
    # unit scales everywhere but one (row, K-block) of A and one (N-block, K-block) of B
    p = inputs.dense_fp8_problem(256, 448, 512, seed=12)
    sfa = np.full_like(p["sfa"], 127)
    sfb = np.full_like(p["sfb"], 127)
    sfa[77, 3] = 131
    sfb[2, 1] = 124
    D = ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(sfa), to_dev(p["B"]), to_dev(sfb), sfb_gran_n=128)
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), orc.gemm_fp8(p["A"], sfa, p["B"], sfb), "single-scale")


# ------------------------------------------------------------------ BF16 / FP4

@pytest.mark.parametrize("m,n,k", [(256, 448, 512), (130, 200, 200), (128, 224, 64), (300, 1000, 1000)])
def test_bf16(ops, orc, m, n, k):
    p = inputs.dense_bf16_problem(m, n, k, seed=m)
    A = to_dev(p["A"], torch.bfloat16)
    B = to_dev(p["B"], torch.bfloat16)
    ldd = (n + 7) // 8 * 8
    D = torch.empty((m, ldd), dtype=torch.bfloat16, device="cuda")[:, :n]
    ops.gemm_bf16_nt(A, B, D)
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), orc.gemm_bf16(p["A"], p["B"]), f"bf16 {m}x{n}x{k}")


def test_bf16_identity_bit_exact(ops, orc):
    k = 128
    eye = np.zeros((k, k), np.float32)
    eye[np.arange(k), np.arange(k)] = 1.0
    A = inputs.bf16_operand(eye)
    B = inputs.bf16_operand(np.random.default_rng(1).standard_normal((224, k)).astype(np.float32))
    D = ops.gemm_bf16_nt(to_dev(A, torch.bfloat16), to_dev(B, torch.bfloat16))
    _status_ok(ops)
    assert np.array_equal(D.view(torch.int16).cpu().numpy().view(np.uint16), B.T)


@pytest.mark.parametrize("m,n,k", [(256, 448, 1024), (130, 250, 320), (128, 224, 64), (256, 512, 4096)])
def test_fp4(ops, orc, m, n, k):
    p = inputs.dense_fp4_problem(m, n, k, seed=n)
    ldd = (n + 7) // 8 * 8
    D = torch.empty((m, ldd), dtype=torch.bfloat16, device="cuda")[:, :n]
    ops.gemm_fp4_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]), D)
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), orc.gemm_fp4(p["A"], p["sfa"], p["B"], p["sfb"]), f"fp4 {m}x{n}x{k}")


# ------------------------------------------------------------------ small M, transposed

@pytest.mark.parametrize("m,n,k,gran", [(128, 7168, 2048, 128), (77, 1000, 1024, 1), (1, 4000, 640, 128),
                                        (33, 300, 4096, 1), (128, 256, 128, 128)])
def test_fp8_small_m_runs_transposed(ops, orc, m, n, k, gran):
    # M <= 128: D^T = B A^T on 256 x 128 pair tiles, written back transposed; ragged N and M,
    # per-row and 128x128 B scales, split and unsplit plans
    plan = ops.gemm_plan("fp8", m, n, k)
    assert plan["transposed"] == 1 and plan["tile_m"] == 256 and plan["tile_n"] == 128, plan
    _fp8_case(ops, orc, m, n, k, seed=m * 13 + n, gran=gran)


# M <= 128 whose transposed tiles are all cut into two K slices: the two halves run on the two
# CTA pairs of a 4-CTA cluster and meet in distributed shared memory (ragged N along the tile rows,
# M below 32 and not a multiple of 8, per-row and 128x128 B scales)
@pytest.mark.parametrize("m,n,k,gran", [(128, 7168, 2048, 128), (100, 5000, 2048, 1), (17, 7000, 4096, 128),
                                        (128, 1024, 2048, 1)])
def test_fp8_small_m_cluster_split(ops, orc, m, n, k, gran):
    plan = ops.gemm_plan("fp8", m, n, k)
    assert plan["cluster_split"] == 1 and plan["splits"] == 2 and plan["transposed"] == 1, plan
    _fp8_case(ops, orc, m, n, k, seed=m * 3 + n, gran=gran)
    p = inputs.dense_fp8_problem(m, n, k, seed=5, b_block_rows=gran)
    args = [to_dev(p[x]) for x in ("A", "sfa", "B", "sfb")]
    d1 = ops.gemm_fp8_nt(*args, sfb_gran_n=gran)
    d2 = ops.gemm_fp8_nt(*args, sfb_gran_n=gran)
    _status_ok(ops)
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


# The same cluster split for BF16 and FP4 (FP4 carrying its scale chunks every K step)
@pytest.mark.parametrize("kind,m,n,k", [("bf16", 64, 7000, 1024), ("bf16", 128, 6500, 2048), ("fp4", 40, 6500, 4096),
                                        ("fp4", 128, 7168, 4096)])
def test_bf16_fp4_small_m_cluster_split(ops, orc, kind, m, n, k):
    plan = ops.gemm_plan(kind, m, n, k)
    assert plan["cluster_split"] == 1 and plan["splits"] == 2 and plan["transposed"] == 1, plan
    got, ref = _run_kind(ops, kind, m, n, k, seed=m + n + k)
    check_gemm(got, ref(orc), f"{kind} cluster split {m}x{n}x{k}")
    again, _ = _run_kind(ops, kind, m, n, k, seed=m + n + k)
    assert np.array_equal(got, again)


@pytest.mark.parametrize("kind,m,n,k", [("bf16", 128, 3000, 2048), ("bf16", 5, 448, 640), ("fp4", 128, 2000, 4096),
                                        ("fp4", 40, 704, 1024)])
def test_bf16_fp4_small_m_run_transposed(ops, orc, kind, m, n, k):
    plan = ops.gemm_plan(kind, m, n, k)
    assert plan["transposed"] == 1 and plan["tile_n"] == 128, plan
    got, ref = _run_kind(ops, kind, m, n, k, seed=m + n)
    check_gemm(got, ref(orc), f"{kind} small M {m}x{n}x{k} {plan}")


# ------------------------------------------------------------------ split last wave

def _run_kind(ops, kind, m, n, k, seed, gran=128, rows=None, cols=None):
    """Run one GEMM on the GPU and return (D as f64, oracle value on rows x cols)."""
    ldd = (n + 7) // 8 * 8
    D = torch.empty((m, ldd), dtype=torch.bfloat16, device="cuda")[:, :n]
    orc_args = dict(rows=rows, cols=cols) if rows is not None else {}
    if kind == "fp8":
        p = inputs.dense_fp8_problem(m, n, k, seed=seed, b_block_rows=gran)
        ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]), D, sfb_gran_n=gran)
        ref = lambda orc: orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=gran, **orc_args)
    elif kind == "fp4":
        p = inputs.dense_fp4_problem(m, n, k, seed=seed)
        ops.gemm_fp4_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]), D)
        ref = lambda orc: orc.gemm_fp4(p["A"], p["sfa"], p["B"], p["sfb"], **orc_args)
    else:
        p = inputs.dense_bf16_problem(m, n, k, seed=seed)
        ops.gemm_bf16_nt(to_dev(p["A"], torch.bfloat16), to_dev(p["B"], torch.bfloat16), D)
        ref = lambda orc: orc.gemm_bf16(p["A"], p["B"], **orc_args)
    _status_ok(ops)
    got = bf16_to_f64(D)
    if rows is not None:
        got = got[np.ix_(rows, cols)]
    return got, ref


# Shapes whose tiles are fewer than the workers: every tile is cut along K into slices whose
# fp32 partial sums are added in a workspace; ragged M / N, uneven slices (K = 2560: five
# scale groups in two slices) and a partial last scale group (K = 2688) included.
@pytest.mark.parametrize("kind,m,n,k,gran", [("fp8", 256, 1024, 4096, 128), ("fp8", 300, 1000, 2560, 128),
                                             ("fp8", 300, 1000, 2688, 1), ("bf16", 256, 512, 4096, 1),
                                             ("bf16", 130, 1000, 4096, 1), ("fp4", 256, 512, 8192, 1)])
def test_split_tiles_every_output(ops, orc, kind, m, n, k, gran):
    plan = ops.gemm_plan(kind, m, n, k)
    assert plan["splits"] > 1 and plan["split_tiles"] * plan["splits"] == plan["work_items"], plan
    got, ref = _run_kind(ops, kind, m, n, k, seed=m + k, gran=gran)
    check_gemm(got, ref(orc), f"{kind} split {m}x{n}x{k} {plan}")


# More tiles than workers: whole tiles in full waves, the remainder split; the oracle checks a
# sample of rows and columns that meets every tile.
@pytest.mark.parametrize("kind,m,n,k", [("fp8", 2560, 2048, 2048), ("bf16", 2560, 2048, 1024),
                                        ("fp4", 2560, 2048, 4096)])
def test_split_last_wave_sampled(ops, orc, kind, m, n, k):
    plan = ops.gemm_plan(kind, m, n, k)
    assert plan["splits"] > 1 and plan["work_items"] > plan["split_tiles"] * plan["splits"], plan
    rng = np.random.default_rng(k)
    tm, tn = plan["tile_m"], plan["tile_n"]
    rows = np.unique(np.concatenate([rng.integers(r, min(r + tm, m), 6) for r in range(0, m, tm)])).astype(np.int32)
    cols = np.unique(np.concatenate([rng.integers(c, min(c + tn, n), 6) for c in range(0, n, tn)])).astype(np.int32)
    got, ref = _run_kind(ops, kind, m, n, k, seed=7, rows=rows, cols=cols)
    check_gemm(got, ref(orc), f"{kind} last wave {m}x{n}x{k} {plan}")


# Slice counts that are not powers of two: the rows of each epilogue warp are cut into shares
# of different sizes, some needing two gather passes, and in the transposed kernel the shares
# start at unaligned positions of D's rows.
@pytest.mark.parametrize("kind,m,n,k,gran,splits", [("fp8", 512, 2560, 3072, 128, 3), ("fp8", 96, 3584, 5120, 1, 5),
                                                    ("bf16", 64, 1792, 6144, 1, 10),
                                                    ("fp4", 256, 2560, 16384, 1, 7)])
def test_split_any_slice_count(ops, orc, kind, m, n, k, gran, splits):
    plan = ops.gemm_plan(kind, m, n, k)
    assert plan["splits"] == splits, plan
    rng = np.random.default_rng(n)
    rows = np.arange(m, dtype=np.int32)  # every row: every share of every warp
    cols = np.unique(np.concatenate([rng.integers(c, min(c + 128, n), 5) for c in range(0, n, 128)])).astype(np.int32)
    if m * n * k <= 2 ** 33:
        rows, cols = None, None
    got, ref = _run_kind(ops, kind, m, n, k, seed=m + n, gran=gran, rows=rows, cols=cols)
    check_gemm(got, ref(orc), f"{kind} {splits} slices {m}x{n}x{k} {plan}")


def test_split_tails_on_two_concurrent_streams(ops, orc):
    # two split-tail GEMMs enqueued on two streams at once: neither waits on a CTA of the other,
    # and a slice never waits on an unscheduled slice of its own tile
    probs = [inputs.dense_fp8_problem(256, 1024, 4096, seed=s) for s in (41, 42)]
    assert ops.gemm_plan("fp8", 256, 1024, 4096)["splits"] > 1
    devs = [[to_dev(p[x]) for x in ("A", "sfa", "B", "sfb")] for p in probs]
    outs = [torch.empty((256, 1024), dtype=torch.bfloat16, device="cuda") for _ in probs]
    streams = [torch.cuda.Stream() for _ in probs]
    torch.cuda.synchronize()
    for _ in range(3):
        for d, o, st in zip(devs, outs, streams):
            with torch.cuda.stream(st):
                ops.gemm_fp8_nt(*d, o)
    torch.cuda.synchronize()
    _status_ok(ops)
    for p, o in zip(probs, outs):
        check_gemm(bf16_to_f64(o), orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"]), "concurrent split")


def test_split_is_deterministic(ops):
    # slices are added in a fixed order, so repeated runs give identical bytes
    p = inputs.dense_fp8_problem(256, 1024, 4096, seed=5)
    args = [to_dev(p[x]) for x in ("A", "sfa", "B", "sfb")]
    d1 = ops.gemm_fp8_nt(*args)
    d2 = ops.gemm_fp8_nt(*args)
    _status_ok(ops)
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


def test_cuda_graph_capture_replays_the_same_bytes(ops):
    # the calls are capturable: scratch becomes a graph memory node, launches become kernel
    # nodes; a replay on new inputs (copied into the captured buffers) matches an eager call
    p = inputs.dense_fp8_problem(512, 1024, 4096, seed=21)
    q = inputs.dense_fp8_problem(512, 1024, 4096, seed=22)
    dv = {x: to_dev(p[x]) for x in ("A", "sfa", "B", "sfb")}
    sa, sb = ops.transform_sf_ue8m0(dv["sfa"]), ops.transform_sf_ue8m0(dv["sfb"])
    D = torch.empty((512, 1024), dtype=torch.bfloat16, device="cuda")
    ops.gemm_fp8_nt(dv["A"], sa, dv["B"], sb, D)  # first call outside capture sets the kernels up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.transform_sf_ue8m0(dv["sfa"], out=sa)
        ops.transform_sf_ue8m0(dv["sfb"], out=sb)
        ops.gemm_fp8_nt(dv["A"], sa, dv["B"], sb, D)
    for x in ("A", "sfa", "B", "sfb"):
        dv[x].copy_(to_dev(q[x]))
    g.replay()
    torch.cuda.synchronize()
    _status_ok(ops)
    eager = ops.gemm_fp8_nt(*[to_dev(q[x]) for x in ("A", "sfa", "B", "sfb")])
    _status_ok(ops)
    assert torch.equal(D.view(torch.int16), eager.view(torch.int16))


# ------------------------------------------------------------------ grouped

def _grouped(ops, p):
    return ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]),
                                                to_dev(p["sfb"]), to_dev(p["m_indices"]))


@pytest.mark.parametrize("counts,n,k", [([100, 0, 150, 50], 448, 512), ([128, 256, 1, 127, 300], 256, 384)])
def test_grouped(ops, orc, counts, n, k):
    p = inputs.grouped_fp8_problem(len(counts), sum(counts), n, k, seed=len(counts), counts=counts)
    D = _grouped(ops, p)
    _status_ok(ops)
    got = bf16_to_f64(D)
    ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"])
    check_gemm(got, ref, "grouped")
    pad = p["m_indices"] < 0
    assert np.all(got[pad] == 0.0)  # padding rows are exactly zero


# N = 448 runs on 224-wide pair tiles (two exactly); N = 512 and N = 1000 on 256-wide ones (the
# latter with a ragged last tile), the accumulator then single-buffered
@pytest.mark.parametrize("n,tile_n", [(448, 224), (512, 256), (1000, 256)])
def test_grouped_pair_tiles_odd_and_even_runs(ops, orc, n, tile_n):
    # experts with 1, 2, 3, 1, 2, 0 and 5 blocks of 128 rows: pairs of blocks of one expert run on
    # CTA pairs, an odd last block alone (its peer CTA's rows, the next expert's, are not written)
    counts = [100, 256, 300, 1, 129, 0, 600]
    p = inputs.grouped_fp8_problem(len(counts), sum(counts), n, 512, seed=23, counts=counts)
    plan = ops.gemm_plan("grouped_fp8", p["M"], n, 512)
    assert plan["tile_m"] == 256 and plan["tile_n"] == tile_n, plan
    D = _grouped(ops, p)
    _status_ok(ops)
    got = bf16_to_f64(D)
    check_gemm(got, orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"]), "grouped pair tiles")
    assert np.all(got[p["m_indices"] < 0] == 0.0)


def test_grouped_beyond_the_pair_list_runs_single_cta(ops, orc):
    # more than 2048 blocks of 128 rows: the single-CTA grouped kernel (128 x 224 tiles)
    counts = [2048 * 128 - 50, 128 + 50, 70]
    n, k = 64, 128
    p = inputs.grouped_fp8_problem(3, sum(counts), n, k, seed=29, counts=counts)
    assert p["M"] // 128 > 2048
    assert ops.gemm_plan("grouped_fp8", p["M"], n, k)["tile_m"] == 128
    D = _grouped(ops, p)
    _status_ok(ops)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([rng.choice(p["M"], 300, replace=False),
                                     np.arange(p["M"] - 400, p["M"])])).astype(np.int32)
    got = bf16_to_f64(D[torch.from_numpy(rows).long().cuda()])
    ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"], rows=rows)
    check_gemm(got, ref, "grouped, single-CTA tiles")


def test_grouped_padding_rows_zero_whatever_a_holds(ops, orc):
    p = inputs.grouped_fp8_problem(2, 200, 224, 256, seed=5, counts=[70, 130])
    p["A"][p["m_indices"] < 0] = 0x38
    got = bf16_to_f64(_grouped(ops, p))
    _status_ok(ops)
    assert np.all(got[p["m_indices"] < 0] == 0.0)
    check_gemm(got, orc.gemm_grouped_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["m_indices"]), "grouped pad")


def test_grouped_single_expert_equals_dense(ops):
    p = inputs.grouped_fp8_problem(1, 384, 448, 512, seed=8, counts=[384])
    Dg = _grouped(ops, p)
    Dd = ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"][0]), to_dev(p["sfb"][0]))
    _status_ok(ops)
    assert torch.equal(Dg.view(torch.int16), Dd.view(torch.int16))


def test_grouped_bad_index_is_flagged(ops):
    p = inputs.grouped_fp8_problem(2, 256, 224, 256, seed=6, counts=[128, 128])
    p["m_indices"][128] = 7  # block start names an expert that does not exist
    _grouped(ops, p)
    assert ops.device_status() == -7
    _status_ok(ops)


# ------------------------------------------------------------------ masked grouped

_SENTINEL = 0x3C5A  # a bf16 bit pattern no product of these inputs is likely to round to exactly


def _masked(ops, p, D=None):
    g, max_m, n = p["G"], p["max_m"], p["N"]
    if D is None:
        D = torch.full((g, max_m, n), 0, dtype=torch.int16, device="cuda").fill_(_SENTINEL).view(torch.bfloat16)
    ops.m_grouped_gemm_fp8_nt_masked(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]),
                                     to_dev(p["masked_m"]), D)
    return D


def _check_masked(orc, p, D, what):
    g, max_m, n = p["G"], p["max_m"], p["N"]
    got = bf16_to_f64(D).reshape(g * max_m, n)
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16).reshape(g * max_m, n)
    valid = np.concatenate([np.arange(max_m) < c for c in p["masked_m"]])
    assert (raw[~valid] == _SENTINEL).all(), f"{what}: rows past masked_m were written"
    if valid.sum() * n >= 1000:
        ref = orc.gemm_masked_fp8(p["A"], p["sfa"], p["B"], p["sfb"], p["masked_m"])
        check_gemm(got[valid], ref[valid], what)


@pytest.mark.parametrize("counts,n,k", [([0, 256, 37, 129], 448, 512), ([1, 128, 255, 64, 0, 200], 1000, 1024)])
def test_masked(ops, orc, counts, n, k):
    p = inputs.masked_fp8_problem(len(counts), 256, n, k, seed=len(counts), counts=counts)
    D = _masked(ops, p)
    _status_ok(ops)
    _check_masked(orc, p, D, f"masked {counts}")


# Transposed masked tiles: an expert's rows in chunks of up to 256 as the MMA's N, cut to the
# chunk's valid rows rounded up to 16 (counts on and off those boundaries, several chunks per
# expert, a ragged N, one and two 128-row atoms of A's scales per chunk).
@pytest.mark.parametrize("counts,max_m,n,k", [([0, 1, 16, 17, 255, 256, 257, 300, 512], 512, 1000, 512),
                                             ([129, 128, 3], 128, 704, 1024), ([200, 64], 384, 256, 256)])
def test_masked_transposed_chunks(ops, orc, counts, max_m, n, k):
    plan = ops.gemm_plan("masked_fp8", max_m, n, k)
    assert plan["transposed"] == 1 and plan["tile_m"] == 256 and plan["tile_n"] == 256, plan
    counts = [min(c, max_m) for c in counts]
    p = inputs.masked_fp8_problem(len(counts), max_m, n, k, seed=sum(counts), counts=counts)
    D = _masked(ops, p)
    _status_ok(ops)
    _check_masked(orc, p, D, f"masked transposed {counts} max_m {max_m}")


def test_masked_random_counts(ops, orc):
    p = inputs.masked_fp8_problem(16, 384, 640, 768, seed=77)
    D = _masked(ops, p)
    _status_ok(ops)
    _check_masked(orc, p, D, "masked random counts")


def test_masked_all_empty_writes_nothing(ops):
    p = inputs.masked_fp8_problem(3, 128, 256, 256, seed=2, counts=[0, 0, 0])
    D = _masked(ops, p)
    _status_ok(ops)
    assert (D.view(torch.int16) == _SENTINEL).all()


def test_masked_equals_contiguous_bit_exact(ops):
    # the same rows through the contiguous layout (each 128-row slab one expert, rows past the
    # count marked -1) run the same MMAs in the same order: identical bytes on the valid rows
    counts = [1, 128, 77, 5]
    p = inputs.masked_fp8_problem(4, 128, 448, 1024, seed=9, counts=counts)
    Dm = _masked(ops, p)
    idx = np.concatenate([np.where(np.arange(128) < c, g, -1) for g, c in enumerate(counts)]).astype(np.int32)
    Dc = ops.m_grouped_gemm_fp8_nt_contiguous(to_dev(p["A"].reshape(512, 1024)), to_dev(p["sfa"]), to_dev(p["B"]),
                                              to_dev(p["sfb"]), to_dev(idx))
    _status_ok(ops)
    valid = torch.from_numpy(idx >= 0).cuda()
    assert torch.equal(Dm.reshape(512, 448)[valid].view(torch.int16), Dc[valid].view(torch.int16))


def test_masked_counts_are_read_on_the_device(ops, orc):
    # capture once, then change the counts on the device between replays
    p = inputs.masked_fp8_problem(4, 256, 448, 512, seed=31, counts=[10, 0, 256, 130])
    dv = {x: to_dev(p[x]) for x in ("A", "sfa", "B", "sfb", "masked_m")}
    sa = ops.transform_sf_ue8m0(dv["sfa"])
    sb = torch.stack([ops.transform_sf_ue8m0(dv["sfb"][e]) for e in range(4)])
    D = torch.empty((4, 256, 448), dtype=torch.bfloat16, device="cuda")
    ops.m_grouped_gemm_fp8_nt_masked(dv["A"], sa, dv["B"], sb, dv["masked_m"], D)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.m_grouped_gemm_fp8_nt_masked(dv["A"], sa, dv["B"], sb, dv["masked_m"], D)
    for counts in ([10, 0, 256, 130], [256, 3, 0, 129]):
        dv["masked_m"].copy_(torch.tensor(counts, dtype=torch.int32))
        D.view(torch.int16).fill_(_SENTINEL)
        g.replay()
        torch.cuda.synchronize()
        _status_ok(ops)
        q = dict(p, masked_m=np.array(counts, np.int32))
        _check_masked(orc, q, D, f"replay {counts}")


def test_masked_bad_count_is_flagged(ops):
    p = inputs.masked_fp8_problem(2, 128, 256, 256, seed=4, counts=[5, 7])
    q = dict(p, masked_m=np.array([5, 300], np.int32))  # 300 > max_m: clamped to 128 and flagged
    _masked(ops, q)
    assert ops.device_status() == -7
    _status_ok(ops)


# ------------------------------------------------------------------ failure detection

def test_wait_timeout_is_reported_and_context_survives(ops, orc):
    # a 2 us wait limit cannot hold whole 256 x 256 x 8192 tiles (40 tiles: too many to split
    # along K): the epilogue's wait for the accumulator runs out and the kernel winds down
    m, n, k = 1280, 2048, 8192
    assert ops.gemm_plan("fp8", m, n, k)["splits"] == 1
    big = inputs.dense_fp8_problem(m, n, k, seed=4)
    args = [to_dev(big[x]) for x in ("A", "sfa", "B", "sfb")]
    old = ops.set_wait_timeout_ns(2000)
    try:
        ops.gemm_fp8_nt(*args)
        assert ops.device_status() == -6
    finally:
        ops.set_wait_timeout_ns(old)
    # the context is still usable
    p = inputs.dense_fp8_problem(256, 448, 1024, seed=5)
    D = ops.gemm_fp8_nt(*[to_dev(p[x]) for x in ("A", "sfa", "B", "sfb")])
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"]), "after timeout")


# ------------------------------------------------------------------ tile shapes

@pytest.mark.parametrize("kind", ["fp8", "bf16", "fp4"])
def test_small_m_many_columns(ops, orc, kind):
    # M <= 128 with N = 16640: 65 transposed pair tiles along N, plus split slices
    m, n, k = 96, 16640, 256
    assert ops.gemm_plan(kind, m, n, k)["transposed"] == 1
    if kind == "fp8":
        p = inputs.dense_fp8_problem(m, n, k, seed=77)
        D = ops.gemm_fp8_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]))
        ref = orc.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"])
    elif kind == "bf16":
        p = inputs.dense_bf16_problem(m, n, k, seed=78)
        D = ops.gemm_bf16_nt(to_dev(p["A"], torch.bfloat16), to_dev(p["B"], torch.bfloat16))
        ref = orc.gemm_bf16(p["A"], p["B"])
    else:
        p = inputs.dense_fp4_problem(m, n, k, seed=79)
        D = ops.gemm_fp4_nt(to_dev(p["A"]), to_dev(p["sfa"]), to_dev(p["B"]), to_dev(p["sfb"]))
        ref = orc.gemm_fp4(p["A"], p["sfa"], p["B"], p["sfb"])
    _status_ok(ops)
    check_gemm(bf16_to_f64(D), ref, f"{kind} wide single-CTA")
