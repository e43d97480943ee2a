"""GPU parity of the FP8 block quantiser (quantize_fp8_ue8m0) against the fp64 oracle.

Codes and packed scale words are integers decided from the same fp32 inputs, so they
are compared bit-exactly: every byte of q and every int16 word of the packed scales,
padding words included.  The GPU kernel takes its block exponent from the amax bit
pattern and rounds with cvt.rn.satfinite; the oracle searches the exponent in fp64 and
rounds with rint on the E4M3 grid.
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


def _spread(rows, cols, seed, bf16=False):
    """N(0,1) values with block magnitudes spread over many binades, an all-zero block, a
    negative zero, a block under the UE8M0 floor, and values on E4M3 rounding ties."""
    rng = np.random.default_rng(seed)
    x = inputs.normal_matrix(rows, cols, seed)
    x *= np.ldexp(np.float32(1.0), rng.integers(-60, 60, size=(rows, 1))).astype(np.float32)
    x[0, :128] = 0.0
    x[min(1, rows - 1), 5] = -0.0
    x[-1, -128:] *= np.float32(2.0 ** -100)
    if rows > 2:
        # a block with amax exactly 448 (exponent 0) holding E4M3 rounding ties
        x[2, :128] = rng.standard_normal(128).astype(np.float32)
        x[2, :4] = [448.0, 1.0625, 1.1875, -2.0 ** -10 * 3]
    if bf16:
        return inputs.bf16_operand(x)
    return x


def _check(ops, orc, x, block_rows):
    rows, cols = x.shape
    xt = to_dev(x, torch.bfloat16) if x.dtype == np.uint16 else to_dev(x)
    q, sf = ops.quantize_fp8(xt, block_rows)
    assert ops.device_status() == 0
    q_ref, e_ref = orc.quantize_fp8(x, block_rows)
    assert np.array_equal(q.cpu().numpy(), q_ref), "codes differ"
    sf_ref = orc.sf_pack(e_ref, ld_out=sf.shape[1])
    assert np.array_equal(sf.cpu().numpy(), sf_ref), "packed scale words differ"
    return q, sf, q_ref, e_ref


@pytest.mark.parametrize("rows,cols,bf16", [(37, 384, False), (300, 640, True), (1, 128, False),
                                            (256, 1024, True), (33, 256, False)])
def test_rows_1x128_bit_exact(ops, orc, rows, cols, bf16):
    _check(ops, orc, _spread(rows, cols, seed=rows + cols, bf16=bf16), 1)


@pytest.mark.parametrize("rows,cols,bf16", [(300, 640, False), (128, 128, True), (1, 384, False),
                                            (520, 1024, True)])
def test_blocks_128x128_bit_exact(ops, orc, rows, cols, bf16):
    _check(ops, orc, _spread(rows, cols, seed=rows * 7 + cols, bf16=bf16), 128)


def test_full_size_operands_bit_exact(ops, orc):
    # the headline GEMM's operands before quantisation: A fp32 [4096, 16384] in 1x128 blocks,
    # B bf16 [7168, 16384] in 128x128 blocks
    _check(ops, orc, inputs.normal_matrix(4096, 16384, seed=0), 1)
    _check(ops, orc, inputs.normal_matrix(7168, 16384, seed=1, bf16=True), 128)


def test_quantised_operands_feed_the_gemm(ops, orc):
    # quantise both operands on the GPU, multiply, compare with the oracle GEMM on the
    # oracle's own quantisation of the same values
    m, n, k = 256, 448, 1024
    xa, xb = inputs.normal_matrix(m, k, seed=41), inputs.normal_matrix(n, k, seed=42)
    qa, sa = ops.quantize_fp8(to_dev(xa), 1)
    qb, sb = ops.quantize_fp8(to_dev(xb), 128)
    D = ops.gemm_fp8_nt(qa, sa, qb, sb, sfb_gran_n=128)
    assert ops.device_status() == 0
    ca, ea = orc.quantize_fp8(xa, 1)
    cb, eb = orc.quantize_fp8(xb, 128)
    check_gemm(bf16_to_f64(D), orc.gemm_fp8(ca, ea, cb, eb, gran_n=128), "quantise + gemm")


def test_non_finite_input_is_flagged(ops):
    x = np.ones((64, 256), np.float32)
    x[10, 200] = np.nan
    ops.quantize_fp8(to_dev(x), 1)
    assert ops.device_status() == -7
    x[10, 200] = 1.0
    x[3, 3] = -np.inf
    ops.quantize_fp8(to_dev(x), 128)
    assert ops.device_status() == -7
    ops.quantize_fp8(to_dev(np.ones((64, 256), np.float32)), 1)
    assert ops.device_status() == 0
