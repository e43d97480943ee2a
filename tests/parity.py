"""Shared helpers of the GPU parity tests: uploads and the GEMM tolerance check.

Tolerance (stated for the GEMM outputs against the fp64 oracle value D* before bf16
rounding): relative Frobenius error <= 2e-3 and per-element |D - D*| <= 1e-2 * (|D*| + 1).
bf16 output rounding alone contributes up to 2^-8 relative per element and about 1.5e-3
in Frobenius norm over many elements, so the Frobenius bound is a statement about
outputs of at least ~1000 elements; check_gemm refuses smaller ones (those shapes are
checked bit-exactly through closed forms instead).
"""

from __future__ import annotations

import numpy as np

FROB_TOL = 2e-3
ELEM_TOL = 1e-2


def to_dev(a: np.ndarray, dtype=None):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_to_f64(t) -> np.ndarray:
    import torch

    return t.float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else np.asarray(t, np.float64)


def check_gemm(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Assert the stated GEMM bounds; returns (relative Frobenius error, worst element ratio)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert got.size >= 1000, "the Frobenius bound needs at least ~1000 outputs"
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    frob = np.linalg.norm(err) / (nref if nref > 0 else 1.0)
    ratio = np.abs(err) / (ELEM_TOL * (np.abs(ref) + 1.0))
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        i = np.unravel_index(np.argmax(ratio), ratio.shape)
        raise AssertionError(f"{what}: element {i} got {got[i]} ref {ref[i]} (ratio {worst:.3g}); frob {frob:.3g}")
    assert frob <= FROB_TOL, f"{what}: relative Frobenius error {frob:.3g} > {FROB_TOL}"
    return frob, worst
