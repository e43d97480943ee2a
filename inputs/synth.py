"""Seeded synthetic operands for the block-scaled GEMM workloads.

Recipe (the one every test, the oracle checks and the bench use):

* Values are drawn as fp32 N(0,1) from ``numpy.random.default_rng(seed)``
  (``standard_normal(dtype=float32)``), row by row in chunks so that full-size
  workloads never hold more than a few hundred MB of fp32 at once.
* FP8 operands: E4M3 (finite variant, max 448) with one power-of-two UE8M0 scale
  per block: 1x128 (one row, 128 consecutive K) for activations, 128x128 for
  weights.  The block exponent is the smallest integer ``e`` with
  ``448 * 2**e >= amax`` (exact integer search, no floating log2), i.e. the scale
  ``2**ceil(log2(amax/448))``; an all-zero block gets ``e = 0``.  The biased
  UE8M0 byte is ``e + 127`` clamped to [1, 254].  Values are ``x / 2**e`` (exact,
  the scale is a power of two) rounded to nearest-even E4M3.
* FP4 operands: E2M1 with one UE8M0 scale per 1x32 block (``2**ceil(log2(amax/6))``)
  for both A and B, rounded to nearest-even E2M1, two values per byte with the
  even K index in the low nibble.
* BF16 operands: N(0,1)/sqrt(K) in fp32, rounded to nearest-even bf16.
* Grouped (MoE) rows: ``rng.dirichlet(ones(G))`` proportions of the valid rows,
  integer counts by the largest-remainder rule, each expert segment padded up to
  a multiple of 128 rows.  Padding rows hold zero codes, a unit scale and the
  expert index -1.
* Masked grouped (decode) layout: every expert owns a slab of max_m rows of A and
  D; its valid-row count is drawn uniformly from [0, max_m] (``rng.integers``)
  unless given.  All max_m rows of every slab hold quantised N(0,1) data, so rows
  past the count carry real-looking values that the GEMM must ignore.

The rounding into E4M3 / E2M1 / bf16 uses ``ml_dtypes`` casts (round to nearest,
ties to even); the oracle's own decode tables are built independently from the
formats' bit fields.
"""

from __future__ import annotations

import math

import ml_dtypes
import numpy as np

QMAX_E4M3 = 448.0
QMAX_E2M1 = 6.0

_CHUNK_ROWS = 1024


def ue8m0_exponent_for_amax(amax: np.ndarray, qmax: float) -> np.ndarray:
    """Smallest integer e with qmax * 2**e >= amax (e = 0 where amax == 0).

    Returned unbiased, int32, clamped to the UE8M0 range [-126, 127].
    """
    a = np.asarray(amax, dtype=np.float64)
    _, e0 = np.frexp(a)  # a = f * 2**e0, f in [0.5, 1)
    # qmax * 2**e >= a; start one binade low and walk up/down exactly.
    e = e0.astype(np.int64) - int(math.floor(math.log2(qmax))) - 1
    for _ in range(3):
        e = e + (np.ldexp(qmax, e) < a)
    for _ in range(3):
        e = e - (np.ldexp(qmax, e - 1) >= a)
    e = np.where(a == 0, 0, e)
    return np.clip(e, -126, 127).astype(np.int32)


def _block_amax(x: np.ndarray, block_rows: int, block_k: int) -> np.ndarray:
    r, k = x.shape
    rb = -(-r // block_rows)
    pad = rb * block_rows - r
    ax = np.abs(x)
    if pad:
        ax = np.concatenate([ax, np.zeros((pad, k), ax.dtype)], axis=0)
    return ax.reshape(rb, block_rows, k // block_k, block_k).max(axis=(1, 3))


def _expand_scale(e: np.ndarray, block_rows: int, block_k: int, r: int) -> np.ndarray:
    """Per-element power-of-two scale 2**-e (fp32) broadcast over the blocks."""
    inv = np.ldexp(np.float32(1.0), -e).astype(np.float32)
    inv = np.repeat(np.repeat(inv, block_rows, axis=0)[:r], block_k, axis=1)
    return inv


def quantize_e4m3_blocks(x: np.ndarray, block_rows: int, block_k: int = 128):
    """fp32 [R, K] -> (E4M3 codes uint8 [R, K], biased UE8M0 exponents uint8 [ceil(R/block_rows), K/block_k])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    r, k = x.shape
    if k % block_k:
        raise ValueError("K must be a multiple of the scale block")
    e = ue8m0_exponent_for_amax(_block_amax(x, block_rows, block_k), QMAX_E4M3)
    scaled = x * _expand_scale(e, block_rows, block_k, r)
    codes = scaled.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    return codes, (e + 127).astype(np.uint8)


def quantize_e2m1_blocks(x: np.ndarray, block_k: int = 32):
    """fp32 [R, K] -> (packed E2M1 uint8 [R, K/2], biased UE8M0 exponents uint8 [R, K/block_k])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    r, k = x.shape
    if k % block_k or k % 2:
        raise ValueError("K must be a multiple of the scale block")
    e = ue8m0_exponent_for_amax(_block_amax(x, 1, block_k), QMAX_E2M1)
    scaled = x * _expand_scale(e, 1, block_k, r)
    nib = scaled.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0x0F
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, (e + 127).astype(np.uint8)


def bf16_operand(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def _normal_rows(rng: np.random.Generator, rows: int, k: int):
    """Yield (row0, fp32 block) chunks of N(0,1) values, drawn row-major in order."""
    for r0 in range(0, rows, _CHUNK_ROWS):
        n = min(_CHUNK_ROWS, rows - r0)
        yield r0, rng.standard_normal((n, k), dtype=np.float32)


def normal_matrix(rows: int, k: int, seed: int, bf16: bool = False) -> np.ndarray:
    """Unquantised operand for the quantiser: fp32 N(0,1) [rows, k] from ``default_rng(seed)``
    (the same draw the quantised operands start from), or its bf16 rounding as uint16 bits."""
    rng = np.random.default_rng(seed)
    x = np.empty((rows, k), np.float32)
    for r0, chunk in _normal_rows(rng, rows, k):
        x[r0:r0 + chunk.shape[0]] = chunk
    return bf16_operand(x) if bf16 else x


def _fp8_operand(rows: int, k: int, seed: int, block_rows: int):
    rng = np.random.default_rng(seed)
    codes = np.empty((rows, k), np.uint8)
    exps = np.empty((-(-rows // block_rows), k // 128), np.uint8)
    step = _CHUNK_ROWS  # multiple of 128, so 128-row blocks never straddle chunks
    for r0, x in _normal_rows(rng, rows, k):
        c, e = quantize_e4m3_blocks(x, block_rows)
        codes[r0:r0 + x.shape[0]] = c
        b0 = r0 // block_rows
        exps[b0:b0 + e.shape[0]] = e
    assert step % 128 == 0
    return codes, exps


def dense_fp8_problem(m: int, n: int, k: int, seed: int = 0, b_block_rows: int = 128):
    """FP8 NT problem: A 1x128 scales, B b_block_rows x 128 scales (128 by default)."""
    a, sfa = _fp8_operand(m, k, seed, 1)
    b, sfb = _fp8_operand(n, k, seed + 1, b_block_rows)
    return {"kind": "fp8", "M": m, "N": n, "K": k, "A": a, "sfa": sfa, "B": b, "sfb": sfb,
            "gran_n": b_block_rows}


def dense_fp4_problem(m: int, n: int, k: int, seed: int = 0):
    """FP4 NT problem: E2M1 packed two per byte, 1x32 UE8M0 scales for A and B."""
    out = {"kind": "fp4", "M": m, "N": n, "K": k}
    for name, rows, s in (("A", m, seed), ("B", n, seed + 1)):
        rng = np.random.default_rng(s)
        packed = np.empty((rows, k // 2), np.uint8)
        exps = np.empty((rows, k // 32), np.uint8)
        for r0, x in _normal_rows(rng, rows, k):
            p, e = quantize_e2m1_blocks(x)
            packed[r0:r0 + x.shape[0]] = p
            exps[r0:r0 + x.shape[0]] = e
        out[name] = packed
        out["sf" + name.lower()] = exps
    return out


def dense_bf16_problem(m: int, n: int, k: int, seed: int = 0):
    """BF16 NT problem: N(0,1)/sqrt(K) rounded to bf16 (uint16 bit patterns)."""
    out = {"kind": "bf16", "M": m, "N": n, "K": k}
    inv = np.float32(1.0 / math.sqrt(k))
    for name, rows, s in (("A", m, seed), ("B", n, seed + 1)):
        rng = np.random.default_rng(s)
        bits = np.empty((rows, k), np.uint16)
        for r0, x in _normal_rows(rng, rows, k):
            bits[r0:r0 + x.shape[0]] = bf16_operand(x * inv)
        out[name] = bits
    return out


def dirichlet_segments(rng: np.random.Generator, groups: int, total_rows: int, alpha: float = 1.0):
    """Integer row counts per expert summing to total_rows (largest-remainder rounding)."""
    p = rng.dirichlet(np.full(groups, alpha))
    raw = p * total_rows
    counts = np.floor(raw).astype(np.int64)
    rem = total_rows - int(counts.sum())
    order = np.argsort(-(raw - counts), kind="stable")
    counts[order[:rem]] += 1
    return counts


def grouped_fp8_problem(groups: int, total_rows: int, n: int, k: int, seed: int = 0,
                        alpha: float = 1.0, align: int = 128, counts=None, b_block_rows: int = 128):
    """M-grouped contiguous FP8 problem (MoE): expert segments padded to `align` rows; each
    expert's B has b_block_rows x 128 scale blocks (128 by default, 1 = one scale per row)."""
    rng = np.random.default_rng(seed)
    if counts is None:
        counts = dirichlet_segments(rng, groups, total_rows, alpha)
    counts = np.asarray(counts, dtype=np.int64)
    padded = ((counts + align - 1) // align) * align
    m_total = int(padded.sum())
    a = np.zeros((m_total, k), np.uint8)
    sfa = np.full((m_total, k // 128), 127, np.uint8)
    m_indices = np.full(m_total, -1, np.int32)
    a_codes, a_sf = _fp8_operand(int(counts.sum()), k, seed + 1, 1)
    src = 0
    dst = 0
    for g in range(groups):
        c = int(counts[g])
        a[dst:dst + c] = a_codes[src:src + c]
        sfa[dst:dst + c] = a_sf[src:src + c]
        m_indices[dst:dst + c] = g
        src += c
        dst += int(padded[g])
    del a_codes, a_sf
    b, sfb = _expert_weights(groups, n, k, seed, b_block_rows)
    return {"kind": "grouped_fp8", "G": groups, "M": m_total, "N": n, "K": k, "A": a, "sfa": sfa,
            "B": b, "sfb": sfb, "m_indices": m_indices, "counts": counts, "gran_n": b_block_rows}


def _expert_weights(groups: int, n: int, k: int, seed: int, b_block_rows: int):
    """Per-expert B [G, N, K] and its UE8M0 exponents [G, ceil(N/b_block_rows), K/128]."""
    b = np.empty((groups, n, k), np.uint8)
    sfb = np.empty((groups, -(-n // b_block_rows), k // 128), np.uint8)
    for g in range(groups):
        b[g], sfb[g] = _fp8_operand(n, k, seed + 2 + g, b_block_rows)
    return b, sfb


def masked_fp8_problem(groups: int, max_m: int, n: int, k: int, seed: int = 0, counts=None,
                       b_block_rows: int = 128):
    """Masked grouped FP8 problem: A [G, max_m, K] (1x128 scales, [G*max_m, K/128]),
    B [G, N, K] (b_block_rows x 128 scales, 128 by default), masked_m [G] valid rows per expert."""
    rng = np.random.default_rng(seed)
    if counts is None:
        counts = rng.integers(0, max_m + 1, size=groups)
    masked_m = np.asarray(counts, dtype=np.int32)
    if masked_m.shape != (groups,) or masked_m.min() < 0 or masked_m.max() > max_m:
        raise ValueError("counts must be G values in [0, max_m]")
    a, sfa = _fp8_operand(groups * max_m, k, seed + 1, 1)
    b, sfb = _expert_weights(groups, n, k, seed, b_block_rows)
    return {"kind": "masked_fp8", "G": groups, "max_m": max_m, "N": n, "K": k,
            "A": a.reshape(groups, max_m, k), "sfa": sfa, "B": b, "sfb": sfb, "masked_m": masked_m,
            "gran_n": b_block_rows}
