"""CPU checks of the C-ABI boundary: the library loads, exports every symbol bsp.h
declares, and rejects bad arguments before touching the GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bsp.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|uint64_t|char\s*\*|const char\s*\*)\s*\**\s*(\w+)\s*\(",
                                 src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from block_scaled_precision_sm_b200 import _lib, build

    build.build()
    return _lib.load()


def test_header_declares_the_calls():
    names = _declared()
    for n in ("gemm_bf16_nt", "gemm_fp8_nt", "gemm_fp4_nt", "m_grouped_gemm_fp8_nt_contiguous",
              "transform_sf_ue8m0", "bsp_get_device_status", "bsp_status_string"):
        assert n in names


def test_exports_every_declared_symbol(lib):
    from block_scaled_precision_sm_b200 import _lib

    for n in _declared():
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    from block_scaled_precision_sm_b200 import _lib

    for code in range(-7, 1):
        assert _lib.describe(code)
    assert _lib.describe(123) == "unknown status"


def test_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    good = vp(0x10000)  # never dereferenced: validation fails first
    odd = vp(0x10001)
    # null pointer, empty sizes
    assert lib.gemm_fp8_nt(None, good, good, good, good, 128, 128, 128, 128, 128, 128, 128, 8, 128, None) == -1
    assert lib.gemm_fp8_nt(good, good, good, good, good, 0, 128, 128, 128, 128, 128, 128, 8, 128, None) == -1
    assert lib.gemm_bf16_nt(good, good, good, 128, -1, 64, 64, 64, 64, None) == -1
    # K breaks its rule
    assert lib.gemm_fp8_nt(good, good, good, good, good, 128, 128, 100, 128, 128, 128, 128, 8, 128, None) == -3
    assert lib.gemm_fp4_nt(good, good, good, good, good, 128, 128, 96, 48, 48, 128, 128, 128, None) == -3
    assert lib.gemm_bf16_nt(good, good, good, 128, 128, 12, 16, 16, 128, None) == -3
    # misaligned pointer / leading dimension
    assert lib.gemm_fp8_nt(odd, good, good, good, good, 128, 128, 128, 128, 128, 128, 128, 8, 128, None) == -2
    assert lib.gemm_bf16_nt(good, good, good, 128, 128, 64, 68, 64, 128, None) == -2
    # ld too small
    assert lib.gemm_fp8_nt(good, good, good, good, good, 128, 128, 256, 128, 256, 128, 128, 8, 128, None) == -3
    # bad granularity
    assert lib.gemm_fp8_nt(good, good, good, good, good, 128, 128, 128, 128, 128, 128, 128, 8, 64, None) == -1
    # grouped: M_total not a multiple of 128, G < 1
    assert lib.m_grouped_gemm_fp8_nt_contiguous(good, good, good, good, good, good, 100, 128, 128, 2, 128, 8, 128,
                                                None) == -3
    assert lib.m_grouped_gemm_fp8_nt_contiguous(good, good, good, good, good, good, 128, 128, 128, 0, 128, 8, 128,
                                                None) == -1
    # transform: kind, ld_out, overlap
    assert lib.transform_sf_ue8m0(good, 2, 8, 8, 8, vp(0x20000), 8, None) == -1
    assert lib.transform_sf_ue8m0(good, 1, 8, 8, 8, vp(0x20000), 4, None) == -3
    assert lib.transform_sf_ue8m0(good, 1, 8, 8, 8, vp(0x20000), 12, None) == -2
    assert lib.transform_sf_ue8m0(good, 1, 64, 8, 8, vp(0x10010), 64, None) == -1
    # the pair: kind, ld_out, alignment, and each output against the other output and inputs
    pair = lib.transform_sf_ue8m0_pair
    assert pair(good, 8, 8, vp(0x20000), 8, good, 8, 8, vp(0x30000), 8, 2, 8, None) == -1
    assert pair(good, 8, 8, vp(0x20000), 8, good, 16, 8, vp(0x30000), 8, 1, 8, None) == -3
    assert pair(good, 8, 8, vp(0x20000), 8, good, 8, 8, vp(0x30008), 8, 1, 8, None) == -2
    assert pair(good, 8, 8, vp(0x20000), 8, good, 8, 8, vp(0x20010), 8, 1, 8, None) == -1
    assert pair(vp(0x40000), 64, 8, vp(0x20000), 64, good, 8, 8, vp(0x40010), 8, 1, 8, None) == -1
    # the batch: count, strides too small for a tensor, misaligned output stride, overlap, size
    bat = lib.transform_sf_ue8m0_batched
    assert bat(good, 1, 0, 8, 8, 8, 64, vp(0x200000), 8, 32, None) == -1
    assert bat(good, 1, 4, 8, 8, 8, 63, vp(0x200000), 8, 32, None) == -3
    assert bat(good, 1, 4, 8, 8, 8, 64, vp(0x200000), 8, 31, None) == -3
    assert bat(good, 1, 4, 8, 8, 8, 64, vp(0x200000), 8, 36, None) == -2
    assert bat(good, 1, 4, 8, 8, 8, 64, vp(0x10080), 8, 32, None) == -1
    assert bat(good, 1, 70000, 8, 8, 8, 64, vp(0x20000000), 8, 32, None) == -4
    # masked grouped: max_m not a multiple of 128, G out of range, misaligned counts
    mm = vp(0x40000)
    assert lib.m_grouped_gemm_fp8_nt_masked(good, good, good, good, good, mm, 2, 100, 128, 128, 256, 8, 128,
                                            None) == -3
    assert lib.m_grouped_gemm_fp8_nt_masked(good, good, good, good, good, mm, 0, 128, 128, 128, 256, 8, 128,
                                            None) == -1
    assert lib.m_grouped_gemm_fp8_nt_masked(good, good, good, good, good, mm, 1025, 128, 128, 128, 131200, 8,
                                            128, None) == -4
    assert lib.m_grouped_gemm_fp8_nt_masked(good, good, good, good, good, vp(0x40002), 2, 128, 128, 128, 256, 8,
                                            128, None) == -2
    assert lib.m_grouped_gemm_fp8_nt_masked(good, good, good, good, good, None, 2, 128, 128, 128, 256, 8, 128,
                                            None) == -1
    # quantiser: kind, block rows, cols not a multiple of 128, ld too small, misaligned ld / pointer
    qo, so = vp(0x20000), vp(0x30000)
    assert lib.quantize_fp8_ue8m0(good, 2, 8, 128, 128, 1, qo, 128, so, 8, None) == -1
    assert lib.quantize_fp8_ue8m0(good, 0, 8, 128, 128, 64, qo, 128, so, 8, None) == -1
    assert lib.quantize_fp8_ue8m0(None, 0, 8, 128, 128, 1, qo, 128, so, 8, None) == -1
    assert lib.quantize_fp8_ue8m0(good, 0, 8, 192, 192, 1, qo, 192, so, 8, None) == -3
    assert lib.quantize_fp8_ue8m0(good, 0, 8, 128, 64, 1, qo, 128, so, 8, None) == -3
    assert lib.quantize_fp8_ue8m0(good, 0, 16, 128, 128, 1, qo, 128, so, 8, None) == -3  # ld_sf < rows
    assert lib.quantize_fp8_ue8m0(good, 0, 8, 128, 130, 1, qo, 128, so, 8, None) == -2
    assert lib.quantize_fp8_ue8m0(good, 0, 8, 128, 128, 1, qo, 136, so, 12, None) == -2
    assert lib.quantize_fp8_ue8m0(odd, 0, 8, 128, 128, 1, qo, 128, so, 8, None) == -2


def test_plan_rejects_bad_arguments_without_gpu(lib):
    plan = (ctypes.c_int32 * 8)()
    ptr = ctypes.cast(plan, ctypes.c_void_p)
    assert lib.bsp_gemm_plan(5, 256, 256, 256, ptr) == -1  # no such kind
    assert lib.bsp_gemm_plan(-1, 256, 256, 256, ptr) == -1
    assert lib.bsp_gemm_plan(1, 0, 256, 256, ptr) == -1
    assert lib.bsp_gemm_plan(1, 256, 256, -128, ptr) == -1
    assert lib.bsp_gemm_plan(1, 256, 256, 256, None) == -1


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    from block_scaled_precision_sm_b200 import _lib

    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()


def test_noalloc_scratch_limit_without_gpu(lib):
    # the size check comes before any CUDA call: 13000 rows of A scales at K = 16384 do not fit
    vp = ctypes.c_void_p
    good = vp(0x10000)
    st = vp(0x10004)
    assert lib.gemm_fp8_nt_noalloc(good, good, good, good, good, st, 13000, 7168, 16384, 16384, 16384, 7168,
                                   128, 128, 128, None) == -4
    # 12000 rows fit: the call gets past the size check (and then fails without a GPU)
    assert lib.gemm_fp8_nt_noalloc(good, good, good, good, good, st, 12000, 7168, 16384, 16384, 16384, 7168,
                                   128, 128, 128, None) != -4


def test_binding_refuses_host_tensors():
    import torch

    from block_scaled_precision_sm_b200 import ops

    a = torch.zeros((128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        ops.gemm_bf16_nt(a, a)
    with pytest.raises(ValueError, match="CUDA device"):
        ops.quantize_fp8(torch.zeros((4, 128)), 1)
    with pytest.raises(ValueError, match="CUDA device"):
        ops.transform_sf_ue8m0(torch.zeros((4, 2), dtype=torch.uint8))
