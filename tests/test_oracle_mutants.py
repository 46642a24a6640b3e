"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

Every mutant is compiled on the CPU from an edited copy of moe_oracle.c and the
pin suite (test_oracle.py) is run against it in a subprocess; the suite must
fail for every mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "swapped_nibbles": ("int lo = blk[2 + i] & 0x0f;\n        int hi = blk[2 + i] >> 4;",
                        "int hi = blk[2 + i] & 0x0f;\n        int lo = blk[2 + i] >> 4;"),
    "offset_7_not_8": ("out[i] = (double)(lo - 8) * dd;", "out[i] = (double)(lo - 7) * dd;"),
    "dropped_cubic": ("(z + 0.044715 * z * z * z)", "(z)"),
    "gate_up_swapped": ("double g = q4_0_row_dot(gate_up_e + (size_t)c * gu_row, xv, d);\n"
                        "        double u = q4_0_row_dot(gate_up_e + (size_t)(f + c) * gu_row, xv, d);",
                        "double u = q4_0_row_dot(gate_up_e + (size_t)c * gu_row, xv, d);\n"
                        "        double g = q4_0_row_dot(gate_up_e + (size_t)(f + c) * gu_row, xv, d);"),
    "no_expert_scale": ("s += w[(size_t)t * k + j] * (double)expert_scale[e] *",
                        "s += w[(size_t)t * k + j] * (double)(e >= 0) *"),
    "ties_to_higher": ("if (best < 0 || v > bv) {", "if (best < 0 || v >= bv) {"),
    "no_router_scale": ("w[(size_t)t * k + j] = router_scale * exp(", "w[(size_t)t * k + j] = exp("),
    "fp16_exp_bias": ("ldexp((double)(1024 + man), ex - 25)", "ldexp((double)(1024 + man), ex - 24)"),
    "unstable_perm": ("for (long s = 0; s < S; ++s) {\n        int e = ids[s];",
                      "for (long s = S - 1; s >= 0; --s) {\n        int e = ids[s];"),
    "router_transposed": ("(double)router_w[(size_t)e * d + i]", "(double)router_w[(size_t)i * E + e]"),
    "dense_subtracted": ("out[i] += dense[i];", "out[i] -= dense[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-w", "-fopenmp", "-fPIC", "-shared",
                    "-o", str(so), str(msrc), "-lm"], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
