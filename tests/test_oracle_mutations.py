"""Plant plausible mistakes in a copy of the oracle and check the pins catch each one.

Every mutant is a text edit of oracle.c compiled in a temporary directory; the
pin suites (test_oracle_pins.py, test_inputs.py) run against it in a child
process and must fail.  The real oracle is never modified.
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "e4m3_bias": ("(int)e - 7", "(int)e - 8"),
    "e4m3_subnormal_exp": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "e2m1_bias": ("(int)e - 1);", "(int)e - 2);"),
    "ue8m0_bias": ("(int)code - 127", "(int)code - 128"),
    "fp4_nibble_order": ("(a[k / 2] >> ((k % 2) * 4))", "(a[k / 2] >> ((1 - k % 2) * 4))"),
    "dropped_b_scale": ("acc += T_UE8M0[sa[kb]] * T_UE8M0[sb[kb]] * s;", "acc += T_UE8M0[sa[kb]] * s;"),
    "dropped_last_block": ("for (int kb = 0; kb < K / 128; ++kb) {", "for (int kb = 0; kb < K / 128 - 1; ++kb) {"),
    "wrong_operand": ("s += T_E4M3[a[k]] * T_E4M3[b[k]];", "s += T_E4M3[a[k]] * T_E4M3[a[k]];"),
    "b_scale_granularity": ("sfb + (int64_t)(n / gran_n) * KB, K);\n        }", "sfb + (int64_t)(n / 128) * KB, K);\n        }"),
    "sf_pack_byte_order": ("v = (uint16_t)(lo | (hi << 8));", "v = (uint16_t)(hi | (lo << 8));"),
    "bf16_truncates": ("q = ldexp(rint(ldexp(x, -lsb)), lsb);", "q = ldexp(trunc(ldexp(x, -lsb)), lsb);"),
    "padding_rows_use_expert0": ("int g = m_indices[m];", "int g = m_indices[m] < 0 ? 0 : m_indices[m];"),
    "quant_exponent_one_low": ("while (ldexp(qmax, e) < amax) ++e;", "while (ldexp(qmax, e + 1) < amax) ++e;"),
    "quant_truncates": ("double r = rint(a / step) * step;", "double r = trunc(a / step) * step;"),
    "quant_ties_away": ("double r = rint(a / step) * step;", "double r = round(a / step) * step;"),
    "quant_drops_sign": ("unsigned s = signbit(v) ? 0x80u : 0u;", "unsigned s = v < 0.0 ? 0x80u : 0u;"),
    "quant_block_first_row_only": ("for (int r = r0; r < r1; ++r)\n                for (int c = kb * 128; c < kb * 128 + 128; ++c) {\n                    double a",
                                   "for (int r = r0; r < r0 + 1; ++r)\n                for (int c = kb * 128; c < kb * 128 + 128; ++c) {\n                    double a"),
    "quant_no_clamp": ("if (ex < -126) ex = -126;", "if (ex < -127) ex = -127;"),
    "quant_subnormal_step": ("ldexp(1.0, -9) : ldexp(1.0, E - 3);", "ldexp(1.0, -10) : ldexp(1.0, E - 3);"),
    "masked_expert0_weights": ("B + ((int64_t)g * N + n) * K,", "B + ((int64_t)0 * N + n) * K,"),
    "masked_off_by_one": ("if (m < masked_m[g])", "if (m <= masked_m[g] && m < max_m)"),
    "bf16_sign": ("acc += decode_bf16(A[(int64_t)m * K + k]) * decode_bf16(B[(int64_t)n * K + k]);",
                  "acc -= decode_bf16(A[(int64_t)m * K + k]) * decode_bf16(B[(int64_t)n * K + k]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    shutil.copytree(os.path.join(ROOT, "inputs"), tmp_path / "inputs",
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(tmp_path / "oracle")
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), tmp_path / "oracle" / "__init__.py")
    (tmp_path / "oracle" / "oracle.c").write_text(src.replace(old, new, 1))
    os.makedirs(tmp_path / "tests")
    for f in ("conftest.py", "test_oracle_pins.py", "test_inputs.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "tests"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()
