"""CPU oracle for the block-scaled GEMM and the UE8M0 scale-factor packing.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package; the product path (the CUDA
library and its Python binding) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, decode by table, OpenMP over
output rows); this module only marshals numpy arrays through ctypes.  Every
function states the definition it follows in ``oracle.c``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Werror", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    """Threads the OpenMP loops use (OMP_NUM_THREADS, else the usable cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else len(os.sched_getaffinity(0))


def tables():
    """The decode tables (E4M3 [256], E2M1 [16], UE8M0 [256]) as fp64 arrays."""
    e4, e2, u8 = np.empty(256), np.empty(16), np.empty(256)
    _load().oracle_tables(_p(e4), _p(e2), _p(u8))
    return e4, e2, u8


def sf_pack(e: np.ndarray, ld_out: int | None = None) -> np.ndarray:
    """Biased UE8M0 bytes [MN, KB] -> int16 words [ceil(KB/2), ld_out] (pairs along K, MN-major)."""
    e = _c(e, np.uint8)
    mn, kb = e.shape
    ld_out = mn if ld_out is None else ld_out
    out = np.empty(((kb + 1) // 2, ld_out), np.uint16)
    if _load().oracle_sf_pack(_p(e), mn, kb, ctypes.c_int64(kb), _p(out), ctypes.c_int64(ld_out)):
        raise ValueError("sf_pack: bad arguments")
    return out.view(np.int16)


def sf_unpack(w: np.ndarray, mn: int, kb: int) -> np.ndarray:
    """int16 words [ceil(KB/2), ld] -> biased UE8M0 bytes [MN, KB]."""
    w = _c(w, np.int16).view(np.uint16)
    out = np.empty((mn, kb), np.uint8)
    if _load().oracle_sf_unpack(_p(w), mn, kb, ctypes.c_int64(w.shape[1]), _p(out), ctypes.c_int64(kb)):
        raise ValueError("sf_unpack: bad arguments")
    return out


def fp32_scales_to_ue8m0(s: np.ndarray) -> np.ndarray:
    """Exact positive power-of-two fp32 scales -> biased UE8M0 bytes (ValueError otherwise)."""
    s = _c(s, np.float32)
    out = np.empty(s.shape, np.uint8)
    if _load().oracle_fp32_scales_to_ue8m0(_p(s), ctypes.c_int64(s.size), _p(out)):
        raise ValueError("scale is not an exact positive normal power of two")
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), one round-to-nearest-even step."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_bf16_round(_p(x), ctypes.c_int64(x.size), _p(out))
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sel(rows, cols, m, n):
    r = None if rows is None else _c(rows, np.int32)
    c = None if cols is None else _c(cols, np.int32)
    nr = m if r is None else r.size
    nc = n if c is None else c.size
    return r, c, nr, nc


def gemm_fp8(A, sfa, B, sfb, gran_n=128, rows=None, cols=None) -> np.ndarray:
    """fp64 D[rows][cols] of the FP8 block-scaled NT GEMM.

    A [M,K] E4M3 codes, sfa [M,K/128] biased UE8M0, B [N,K] codes,
    sfb [ceil(N/gran_n), K/128] biased UE8M0.
    """
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.uint8), _c(sfb, np.uint8)
    (m, k), n = A.shape, B.shape[0]
    assert sfa.shape == (m, k // 128) and sfb.shape == (-(-n // gran_n), k // 128)
    r, c, nr, nc = _sel(rows, cols, m, n)
    out = np.empty((nr, nc))
    if _load().oracle_gemm_fp8(_p(A), _p(sfa), _p(B), _p(sfb), gran_n, m, n, k,
                               _p(r), nr, _p(c), nc, _p(out)):
        raise ValueError("gemm_fp8: bad arguments")
    return out


def gemm_fp4(A, sfa, B, sfb, rows=None, cols=None) -> np.ndarray:
    """fp64 D of the FP4 (E2M1, 1x32 UE8M0) NT GEMM; A [M,K/2], B [N,K/2] packed."""
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.uint8), _c(sfb, np.uint8)
    m, k = A.shape[0], A.shape[1] * 2
    n = B.shape[0]
    assert sfa.shape == (m, k // 32) and sfb.shape == (n, k // 32)
    r, c, nr, nc = _sel(rows, cols, m, n)
    out = np.empty((nr, nc))
    if _load().oracle_gemm_fp4(_p(A), _p(sfa), _p(B), _p(sfb), m, n, k, _p(r), nr, _p(c), nc, _p(out)):
        raise ValueError("gemm_fp4: bad arguments")
    return out


def gemm_bf16(A, B, rows=None, cols=None) -> np.ndarray:
    """fp64 D of the BF16 NT GEMM; A [M,K], B [N,K] bf16 bit patterns."""
    A, B = _c(A, np.uint16), _c(B, np.uint16)
    (m, k), n = A.shape, B.shape[0]
    r, c, nr, nc = _sel(rows, cols, m, n)
    out = np.empty((nr, nc))
    if _load().oracle_gemm_bf16(_p(A), _p(B), m, n, k, _p(r), nr, _p(c), nc, _p(out)):
        raise ValueError("gemm_bf16: bad arguments")
    return out


def gemm_grouped_fp8(A, sfa, B, sfb, m_indices, gran_n=128, rows=None, cols=None) -> np.ndarray:
    """fp64 D of the M-grouped contiguous FP8 GEMM; B [G,N,K], sfb [G,ceil(N/gran_n),K/128]."""
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.uint8), _c(sfb, np.uint8)
    idx = _c(m_indices, np.int32)
    (m, k), (g, n) = A.shape, B.shape[:2]
    assert sfb.shape == (g, -(-n // gran_n), k // 128) and idx.shape == (m,)
    r, c, nr, nc = _sel(rows, cols, m, n)
    out = np.empty((nr, nc))
    if _load().oracle_gemm_grouped_fp8(_p(A), _p(sfa), _p(B), _p(sfb), _p(idx), gran_n, g, m, n, k,
                                       _p(r), nr, _p(c), nc, _p(out)):
        raise ValueError("gemm_grouped_fp8: bad arguments (expert index out of range?)")
    return out


def gemm_masked_fp8(A, sfa, B, sfb, masked_m, gran_n=128, rows=None, cols=None) -> np.ndarray:
    """fp64 D [G*max_m (or rows), N (or cols)] of the masked grouped FP8 GEMM: A [G,max_m,K],
    sfa [G*max_m, K/128], B [G,N,K], sfb [G, ceil(N/gran_n), K/128], masked_m [G]; rows of
    expert g at or past masked_m[g] are NaN (not part of the result)."""
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.uint8), _c(sfb, np.uint8)
    mm = _c(masked_m, np.int32)
    (g, max_m, k), n = A.shape, B.shape[1]
    assert B.shape == (g, n, k) and sfa.shape == (g * max_m, k // 128) and mm.shape == (g,)
    assert sfb.shape == (g, -(-n // gran_n), k // 128)
    r, c, nr, nc = _sel(rows, cols, g * max_m, n)
    out = np.empty((nr, nc))
    if _load().oracle_gemm_masked_fp8(_p(A), _p(sfa), _p(B), _p(sfb), _p(mm), gran_n, g, max_m, n, k,
                                      _p(r), nr, _p(c), nc, _p(out)):
        raise ValueError("gemm_masked_fp8: bad arguments (masked_m outside [0, max_m]?)")
    return out


def quantize_fp8(x, block_rows: int = 1):
    """fp32 (or bf16 bit patterns, uint16) [R, K] -> (E4M3 codes uint8 [R, K],
    biased UE8M0 bytes uint8 [ceil(R/block_rows), K/128]); blocks of block_rows x 128."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << 16).view(np.float32)
    x = _c(x, np.float32)
    r, k = x.shape
    q = np.empty((r, k), np.uint8)
    e = np.empty((-(-r // block_rows), k // 128), np.uint8)
    if _load().oracle_quantize_fp8(_p(x), r, k, ctypes.c_int64(k), block_rows, _p(q), _p(e)):
        raise ValueError("quantize_fp8: bad sizes or a non-finite value")
    return q, e
