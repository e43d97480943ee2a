"""ctypes binding of libbsp.so: the C-ABI names and signatures of include/bsp.h, nothing more."""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsp.so")

_vp, _i, _i64, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64

# name -> (restype, argtypes), mirroring include/bsp.h
SIGNATURES = {
    "gemm_bf16_nt": (_i, [_vp, _vp, _vp, _i, _i, _i, _i64, _i64, _i64, _vp]),
    "gemm_fp8_nt": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i64, _i64, _i64, _i64, _i64, _i, _vp]),
    "gemm_fp4_nt": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i64, _i64, _i64, _i64, _i64, _vp]),
    "m_grouped_gemm_fp8_nt_contiguous": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i64, _i64, _i, _vp]),
    "m_grouped_gemm_fp8_nt_masked": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i64, _i64, _i, _vp]),
    "transform_sf_ue8m0": (_i, [_vp, _i, _i, _i, _i64, _vp, _i64, _vp]),
    "transform_sf_ue8m0_pair": (_i, [_vp, _i, _i64, _vp, _i64, _vp, _i, _i64, _vp, _i64, _i, _i, _vp]),
    "transform_sf_ue8m0_batched": (_i, [_vp, _i, _i, _i, _i, _i64, _i64, _vp, _i64, _i64, _vp]),
    "gemm_fp8_nt_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i64, _i64, _i64, _i64, _i64, _i, _vp]),
    "bsp_get_device_status": (_i, [_vp]),
    "bsp_status_string": (ctypes.c_char_p, [_i]),
    "bsp_set_wait_timeout_ns": (_u64, [_u64]),
    "bsp_kernel_launches": (_u64, []),
    "bsp_gemm_plan": (_i, [_i, _i, _i, _i, _vp]),
    "quantize_fp8_ue8m0": (_i, [_vp, _i, _i, _i, _i64, _i, _vp, _i64, _vp, _i64, _vp]),
}

STATUS = {0: "BSP_OK", -1: "BSP_ERR_ARG", -2: "BSP_ERR_ALIGN", -3: "BSP_ERR_SHAPE", -4: "BSP_ERR_UNSUPPORTED",
          -5: "BSP_ERR_CUDA", -6: "BSP_ERR_TIMEOUT", -7: "BSP_ERR_DEVICE_CHECK"}

_lib = None


class BspError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({describe(code)})")


def load() -> ctypes.CDLL:
    """Load libbsp.so (raises if it was not built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with __graft_entry__.build() "
                              "or python block_scaled_precision_sm_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype, f.argtypes = res, args
        _lib = lib
    return _lib


def describe(code: int) -> str:
    return load().bsp_status_string(int(code)).decode()


def call(name: str, *args) -> int:
    rc = getattr(load(), name)(*args)
    if rc != 0:
        raise BspError(name, rc)
    return rc
