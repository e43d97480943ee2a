"""The oracle and the CUDA product path share no code and the product never reaches the
oracle: checked on the sources, so it holds whatever machine the tests run on."""

import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_scaled_precision_sm_b200")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        if "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def test_product_never_imports_the_oracle():
    for path in _files(PKG, (".py",)):
        text = open(path).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), path
        assert "oracle." not in text, path


def test_cuda_sources_and_oracle_include_nothing_of_each_other():
    for path in _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")):
        includes = re.findall(r'#include\s+"([^"]+)"', open(path).read())
        assert not any("oracle" in inc for inc in includes), (path, includes)
    oracle_src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    includes = re.findall(r'#include\s+[<"]([^>"]+)[>"]', oracle_src)
    assert set(includes) <= {"math.h", "stdint.h", "stdlib.h", "string.h"}, includes


def test_inputs_module_holds_no_gemm_or_packing_code():
    # the generators are the only code both sides use; they must not carry the GEMM or the
    # scale packing the two sides compute independently
    text = "".join(open(p).read() for p in _files(os.path.join(ROOT, "inputs"), (".py",)))
    for word in ("matmul", "einsum", "@ ", "sf_pack", "<< 8"):
        assert word not in text, word
