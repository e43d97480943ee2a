"""PyTorch-facing calls of libbsp.so (argument marshalling only).

Every function hands device pointers, sizes and the current CUDA stream to the C ABI
of include/bsp.h; all computation happens in the library's kernels.  Output tensors
are allocated here with torch when the caller does not pass one.

Scale factors: the GEMMs take the packed layout (int16 words, pairs of UE8M0 bytes
along K, MN-major).  ``packed_sf`` implements the "reuse or convert" decision the pages
describe for the scale helper ("DeepGEMM-Ascend cobre quantas operações no Ascend
950?", section "Fatores de escala FP8 e o formato UE8M0 no Ascend"): an int16 tensor
already in that layout is used as it is; fp32 power-of-two scales or uint8 UE8M0
bytes [MN, KB] are converted on the GPU by ``transform_sf_ue8m0``.
"""

from __future__ import annotations

import ctypes
import functools

import torch

from . import _lib


def _on_tensor_device(fn):
    """Run `fn` with its tensors' CUDA device current (the library launches on the current
    device and the current stream); tensors on the CPU or on several devices are refused."""

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        devs = {a.device for a in list(args) + list(kwargs.values()) if isinstance(a, torch.Tensor)}
        if any(d.type != "cuda" for d in devs):
            raise ValueError(f"{fn.__name__}: tensors must live on a CUDA device")
        if len(devs) > 1:
            raise ValueError(f"{fn.__name__}: tensors on several devices: {sorted(map(str, devs))}")
        if not devs:
            return fn(*args, **kwargs)
        with torch.cuda.device(devs.pop()):
            return fn(*args, **kwargs)

    return wrapper


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    if not t.is_cuda:
        raise ValueError("tensor must live on the CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _rowmajor(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with a contiguous last dimension")
    return t.stride(0)


def _bytes_u8(t: torch.Tensor) -> torch.Tensor:
    if t.dtype in (torch.uint8, torch.int8):
        return t.view(torch.uint8)
    if t.element_size() == 1:  # torch.float8_e4m3fn, float4 packed containers
        return t.view(torch.uint8)
    raise ValueError(f"expected a 1-byte dtype, got {t.dtype}")


def sf_ld(mn: int) -> int:
    """Default leading dimension of packed scale words: MN rounded up to 8 (16 bytes)."""
    return (mn + 7) // 8 * 8


@_on_tensor_device
def transform_sf_ue8m0(sf: torch.Tensor, ld_out: int | None = None, stream=None,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 power-of-two scales or uint8 UE8M0 bytes [MN, KB] -> int16 words [ceil(KB/2), ld_out]."""
    ld_in = _rowmajor(sf, "sf")
    mn, kb = sf.shape
    if sf.dtype == torch.float32:
        kind = 0
    elif sf.dtype == torch.uint8:
        kind = 1
    else:
        raise ValueError("scale factors must be float32 (powers of two) or uint8 (UE8M0 bytes)")
    if out is not None:
        ld_out = _rowmajor(out, "out")
        if out.dtype != torch.int16 or out.shape[0] != (kb + 1) // 2 or out.shape[1] < mn:
            raise ValueError("out must be int16 [ceil(KB/2), >= MN]")
    else:
        ld_out = sf_ld(mn) if ld_out is None else ld_out
        out = torch.empty(((kb + 1) // 2, ld_out), dtype=torch.int16, device=sf.device)
    _lib.call("transform_sf_ue8m0", _ptr(sf), kind, mn, kb, ld_in, _ptr(out), ld_out, _stream(stream))
    return out


def _sf_kind(sf: torch.Tensor) -> int:
    if sf.dtype == torch.float32:
        return 0
    if sf.dtype == torch.uint8:
        return 1
    raise ValueError("scale factors must be float32 (powers of two) or uint8 (UE8M0 bytes)")


def _sf_out(out, sf, mn, kb, name):
    if out is None:
        return torch.empty(((kb + 1) // 2, sf_ld(mn)), dtype=torch.int16, device=sf.device)
    _rowmajor(out, name)
    if out.dtype != torch.int16 or out.shape[0] != (kb + 1) // 2 or out.shape[1] < mn:
        raise ValueError(f"{name} must be int16 [ceil(KB/2), >= MN]")
    return out


@_on_tensor_device
def transform_sf_ue8m0_pair(sf_a: torch.Tensor, sf_b: torch.Tensor, out_a: torch.Tensor | None = None,
                            out_b: torch.Tensor | None = None, stream=None):
    """Two transform_sf_ue8m0 conversions with the same dtype and KB (a GEMM's A and B scales)
    in one launch; returns (out_a, out_b)."""
    kind = _sf_kind(sf_a)
    if _sf_kind(sf_b) != kind or sf_a.dim() != 2 or sf_b.dim() != 2 or sf_a.shape[1] != sf_b.shape[1]:
        raise ValueError("sf_a and sf_b must be [MN, KB] of one dtype with the same KB")
    (mn_a, kb), mn_b = sf_a.shape, sf_b.shape[0]
    ld_a, ld_b = _rowmajor(sf_a, "sf_a"), _rowmajor(sf_b, "sf_b")
    out_a, out_b = _sf_out(out_a, sf_a, mn_a, kb, "out_a"), _sf_out(out_b, sf_b, mn_b, kb, "out_b")
    _lib.call("transform_sf_ue8m0_pair", _ptr(sf_a), mn_a, ld_a, _ptr(out_a), out_a.stride(0), _ptr(sf_b), mn_b,
              ld_b, _ptr(out_b), out_b.stride(0), kind, kb, _stream(stream))
    return out_a, out_b


@_on_tensor_device
def transform_sf_ue8m0_batched(sf: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """transform_sf_ue8m0 of every tensor of a stack [G, MN, KB] (fp32 or uint8) in one launch:
    int16 words [G, ceil(KB/2), ld]."""
    kind = _sf_kind(sf)
    if sf.dim() != 3 or sf.stride(2) != 1 or sf.stride(1) < sf.shape[2]:
        raise ValueError("sf must be [G, MN, KB] with KB contiguous")
    g, mn, kb = sf.shape
    if out is None:
        out = torch.empty((g, (kb + 1) // 2, sf_ld(mn)), dtype=torch.int16, device=sf.device)
    if (out.dtype != torch.int16 or out.dim() != 3 or out.shape[0] != g or out.shape[1] != (kb + 1) // 2
            or out.shape[2] < mn or out.stride(2) != 1 or out.stride(1) < out.shape[2]):
        raise ValueError("out must be int16 [G, ceil(KB/2), >= MN] with the last dimension contiguous")
    _lib.call("transform_sf_ue8m0_batched", _ptr(sf), kind, g, mn, kb, sf.stride(1), sf.stride(0), _ptr(out),
              out.stride(1), out.stride(0), _stream(stream))
    return out


def is_packed_sf(sf: torch.Tensor, mn: int, kb: int) -> bool:
    """True if `sf` already is the packed layout for MN scale rows and KB blocks."""
    return (sf.dtype == torch.int16 and sf.dim() == 2 and sf.shape[0] == (kb + 1) // 2
            and sf.shape[1] >= mn and sf.stride(1) == 1 and (sf.stride(0) * 2) % 16 == 0)


@_on_tensor_device
def packed_sf(sf: torch.Tensor, mn: int, kb: int, stream=None) -> torch.Tensor:
    """Reuse `sf` if it already is packed, else convert it (fp32 / uint8 [MN, KB])."""
    if is_packed_sf(sf, mn, kb):
        return sf
    if sf.dim() != 2 or tuple(sf.shape) != (mn, kb):
        raise ValueError(f"scale factors must be packed int16 [{(kb + 1) // 2}, >={mn}] or [{mn}, {kb}]")
    return transform_sf_ue8m0(sf, stream=stream)


def _packed_pair(sfa, mn_a, sfb, mn_b, kb, stream):
    """Both operands' scales packed: each reused if it already is, and converted together in
    one launch when neither is."""
    if (not is_packed_sf(sfa, mn_a, kb) and not is_packed_sf(sfb, mn_b, kb) and sfa.dtype == sfb.dtype
            and sfa.dim() == 2 and tuple(sfa.shape) == (mn_a, kb) and sfb.dim() == 2
            and tuple(sfb.shape) == (mn_b, kb)):
        return transform_sf_ue8m0_pair(sfa, sfb, stream=stream)
    return packed_sf(sfa, mn_a, kb, stream), packed_sf(sfb, mn_b, kb, stream)


def _out(D, m, n, device):
    if D is None:
        return torch.empty((m, n), dtype=torch.bfloat16, device=device)
    if D.dtype != torch.bfloat16 or D.shape[0] != m or D.shape[1] != n:
        raise ValueError("D must be bf16 [M, N]")
    return D


@_on_tensor_device
def gemm_bf16_nt(A: torch.Tensor, B: torch.Tensor, D: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """D = A * B^T for bf16 A [M, K], B [N, K]."""
    if A.dtype != torch.bfloat16 or B.dtype != torch.bfloat16:
        raise ValueError("A and B must be bf16")
    lda, ldb = _rowmajor(A, "A"), _rowmajor(B, "B")
    (m, k), n = A.shape, B.shape[0]
    D = _out(D, m, n, A.device)
    _lib.call("gemm_bf16_nt", _ptr(A), _ptr(B), _ptr(D), m, n, k, lda, ldb, _rowmajor(D, "D"), _stream(stream))
    return D


@_on_tensor_device
def gemm_fp8_nt(A, sfa, B, sfb, D=None, sfb_gran_n: int = 128, stream=None) -> torch.Tensor:
    """FP8 E4M3 block-scaled D = A * B^T.  A [M, K], B [N, K] (1-byte dtypes)."""
    A8, B8 = _bytes_u8(A), _bytes_u8(B)
    lda, ldb = _rowmajor(A8, "A"), _rowmajor(B8, "B")
    (m, k), n = A8.shape, B8.shape[0]
    kb = k // 128
    sfa, sfb = _packed_pair(sfa, m, sfb, -(-n // sfb_gran_n), kb, stream)
    D = _out(D, m, n, A8.device)
    _lib.call("gemm_fp8_nt", _ptr(A8), _ptr(sfa), _ptr(B8), _ptr(sfb), _ptr(D), m, n, k, lda, ldb,
              _rowmajor(D, "D"), sfa.stride(0), sfb.stride(0), sfb_gran_n, _stream(stream))
    return D


@_on_tensor_device
def gemm_fp4_nt(A, sfa, B, sfb, D=None, stream=None) -> torch.Tensor:
    """FP4 E2M1 block-scaled D = A * B^T.  A [M, K/2], B [N, K/2] packed bytes (even K low nibble)."""
    A8, B8 = _bytes_u8(A), _bytes_u8(B)
    lda, ldb = _rowmajor(A8, "A"), _rowmajor(B8, "B")
    m, k, n = A8.shape[0], A8.shape[1] * 2, B8.shape[0]
    kb = k // 32
    sfa, sfb = _packed_pair(sfa, m, sfb, n, kb, stream)
    D = _out(D, m, n, A8.device)
    _lib.call("gemm_fp4_nt", _ptr(A8), _ptr(sfa), _ptr(B8), _ptr(sfb), _ptr(D), m, n, k, lda, ldb,
              _rowmajor(D, "D"), sfa.stride(0), sfb.stride(0), _stream(stream))
    return D


@_on_tensor_device
def m_grouped_gemm_fp8_nt_contiguous(A, sfa, B, sfb, m_indices, D=None, sfb_gran_n: int = 128,
                                     stream=None) -> torch.Tensor:
    """M-grouped FP8 GEMM: A [M_total, K], B [G, N, K], sfb packed per expert [G, words, ld]."""
    A8 = _bytes_u8(A)
    B8 = _bytes_u8(B)
    if not A8.is_contiguous() or not B8.is_contiguous():
        raise ValueError("A and B must be contiguous")
    if m_indices.dtype != torch.int32 or not m_indices.is_contiguous():
        raise ValueError("m_indices must be contiguous int32")
    (m, k), (g, n) = A8.shape, B8.shape[:2]
    kb = k // 128
    sfa = packed_sf(sfa, m, kb, stream)
    mn_b = -(-n // sfb_gran_n)
    if sfb.dim() == 3 and sfb.dtype == torch.int16:
        if sfb.shape[0] != g or sfb.shape[1] != (kb + 1) // 2 or sfb.shape[2] < mn_b or not sfb.is_contiguous():
            raise ValueError("packed sfb must be contiguous int16 [G, words, ld]")
    else:
        if sfb.dim() != 3 or tuple(sfb.shape) != (g, mn_b, kb):
            raise ValueError(f"sfb must be packed int16 [G, words, ld] or [{g}, {mn_b}, {kb}]")
        sfb = transform_sf_ue8m0_batched(sfb, stream=stream)
    D = _out(D, m, n, A8.device)
    if not D.is_contiguous():
        raise ValueError("D must be contiguous")
    _lib.call("m_grouped_gemm_fp8_nt_contiguous", _ptr(A8), _ptr(sfa), _ptr(B8), _ptr(sfb), _ptr(D),
              _ptr(m_indices), m, n, k, g, sfa.stride(0), sfb.stride(1), sfb_gran_n, _stream(stream))
    return D


@_on_tensor_device
def m_grouped_gemm_fp8_nt_masked(A, sfa, B, sfb, masked_m, D=None, sfb_gran_n: int = 128,
                                 stream=None) -> torch.Tensor:
    """Masked grouped FP8 GEMM: A [G, max_m, K], B [G, N, K], masked_m int32 [G] on the device;
    D [G, max_m, N] gets rows m < masked_m[g] of every expert (the other rows are not written)."""
    A8 = _bytes_u8(A)
    B8 = _bytes_u8(B)
    if A8.dim() != 3 or B8.dim() != 3 or not A8.is_contiguous() or not B8.is_contiguous():
        raise ValueError("A [G, max_m, K] and B [G, N, K] must be contiguous")
    if masked_m.dtype != torch.int32 or not masked_m.is_contiguous() or not masked_m.is_cuda:
        raise ValueError("masked_m must be a contiguous int32 device tensor")
    (g, max_m, k), n = A8.shape, B8.shape[1]
    if B8.shape[0] != g or B8.shape[2] != k or masked_m.numel() != g:
        raise ValueError("A, B and masked_m disagree on G or K")
    kb = k // 128
    sfa = packed_sf(sfa.reshape(g * max_m, -1) if sfa.dim() == 3 and sfa.dtype != torch.int16 else sfa,
                    g * max_m, kb, stream)
    mn_b = -(-n // sfb_gran_n)
    if sfb.dim() == 3 and sfb.dtype == torch.int16:
        if sfb.shape[0] != g or sfb.shape[1] != (kb + 1) // 2 or sfb.shape[2] < mn_b or not sfb.is_contiguous():
            raise ValueError("packed sfb must be contiguous int16 [G, words, ld]")
    else:
        if sfb.dim() != 3 or tuple(sfb.shape) != (g, mn_b, kb):
            raise ValueError(f"sfb must be packed int16 [G, words, ld] or [{g}, {mn_b}, {kb}]")
        sfb = transform_sf_ue8m0_batched(sfb, stream=stream)
    if D is None:
        D = torch.empty((g, max_m, n), dtype=torch.bfloat16, device=A8.device)
    if D.dtype != torch.bfloat16 or tuple(D.shape) != (g, max_m, n) or not D.is_contiguous():
        raise ValueError("D must be contiguous bf16 [G, max_m, N]")
    _lib.call("m_grouped_gemm_fp8_nt_masked", _ptr(A8), _ptr(sfa), _ptr(B8), _ptr(sfb), _ptr(D),
              _ptr(masked_m), g, max_m, n, k, sfa.stride(0), sfb.stride(1), sfb_gran_n, _stream(stream))
    return D


def device_status(stream=None) -> int:
    """Synchronise and return (and clear) the status word latched by the kernels."""
    return _lib.load().bsp_get_device_status(_stream(stream))


def set_wait_timeout_ns(ns: int) -> int:
    return int(_lib.load().bsp_set_wait_timeout_ns(int(ns)))


def kernel_launches() -> int:
    return int(_lib.load().bsp_kernel_launches())


@_on_tensor_device
def quantize_fp8(x: torch.Tensor, block_rows: int = 1, q: torch.Tensor | None = None,
                 sf: torch.Tensor | None = None, stream=None):
    """fp32 / bf16 [rows, cols] -> (E4M3 codes uint8 [rows, cols], SF words int16
    [ceil(cols/256), ld]) with one UE8M0 scale per block_rows x 128 block (1 or 128)."""
    if x.dtype == torch.float32:
        kind = 0
    elif x.dtype == torch.bfloat16:
        kind = 1
    else:
        raise ValueError("x must be float32 or bfloat16")
    ld_x = _rowmajor(x, "x")
    rows, cols = x.shape
    scale_rows = -(-rows // block_rows)
    words = (cols // 128 + 1) // 2
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((words, sf_ld(scale_rows)), dtype=torch.int16, device=x.device)
    _lib.call("quantize_fp8_ue8m0", _ptr(x), kind, rows, cols, ld_x, block_rows, _ptr(q), _rowmajor(q, "q"),
              _ptr(sf), _rowmajor(sf, "sf"), _stream(stream))
    return q, sf


_PLAN_KINDS = {"bf16": 0, "fp8": 1, "fp4": 2, "grouped_fp8": 3, "masked_fp8": 4}


def gemm_plan(kind: str, M: int, N: int, K: int) -> dict:
    """How the library would launch this GEMM on the current device (nothing is launched)."""
    out = (ctypes.c_int32 * 8)()
    _lib.call("bsp_gemm_plan", _PLAN_KINDS[kind], M, N, K, ctypes.cast(out, ctypes.c_void_p))
    keys = ("tile_m", "tile_n", "splits", "split_tiles", "work_items", "workers", "transposed", "cluster_split")
    return dict(zip(keys, (int(v) for v in out)))
