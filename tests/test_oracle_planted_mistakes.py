"""The oracle's pins must catch plausible mistakes (CPU only).

Each case copies oracle/oracle.c, plants one mistake by a textual edit (a
dropped term, a wrong sign, index, bias, rounding direction, transposed
layout ...), compiles the copy and runs the oracle pin tests against it in a
child process (FGFP8_ORACLE_LIB points the wrapper at the broken build).  The
pins pass on the real oracle (the other test files) and must fail on every
mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
PIN_TESTS = ["tests/test_oracle_codec.py", "tests/test_oracle_quant.py", "tests/test_oracle_gemm.py",
             "tests/test_oracle_rowcol.py"]

MUTANTS = {
    "tie_to_odd": ("pick = (lo % 2 == 0) ? lo : up;", "pick = (lo % 2 == 0) ? up : lo;"),
    "truncate_not_round": ("if (dlo < dup) pick = lo;", "if (dlo < dup + 1e9) pick = lo;"),
    "exponent_bias_8": ("mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
                        "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "subnormal_exponent": ("mag = ldexp((double)m / 8.0, -6);", "mag = ldexp((double)m / 8.0, -7);"),
    "sign_dropped": ("uint8_t sign = signbit(v) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    "scale_divisor_447": ("float orc_scale_f32(float amax_c) { return amax_c / 448.0f; }",
                          "float orc_scale_f32(float amax_c) { return amax_c / 447.0f; }"),
    "ue8m0_rounds_down": ("int p = (f == 0.5f) ? x - 1 : x;", "int p = x - 1;"),
    "amax_floor_1e-3": ("#define ORC_AMAX_FLOOR 1e-4f", "#define ORC_AMAX_FLOOR 1e-3f"),
    "act_scale_rows_reversed": ("((float*)Xs)[g * ld_s + m] = sf;",
                                "((float*)Xs)[g * ld_s + (M - 1 - m)] = sf;"),
    "weight_amax_first_row_only": ("float amax_c = amax_clamped(blk, ORC_GROUP, ldw, ORC_GROUP);",
                                   "float amax_c = amax_clamped(blk, ORC_GROUP, ldw, 1);"),
    "gemm_weight_scale_dropped": ("y += (sa * sw) * p;", "y += sa * p;"),
    "gemm_weight_scale_transposed": (
        "double sw = scale_at(Ws, ws_off + (n / ORC_GROUP) * KB + kb, fmt);",
        "double sw = scale_at(Ws, ws_off + kb * NB + n / ORC_GROUP, fmt);"),
    "gemm_abs_weight": ("for (int64_t k = kb * ORC_GROUP; k < (kb + 1) * ORC_GROUP; ++k) {\n"
                        "                    double prod = table[xr[k]] * table[wr[k]];",
                        "for (int64_t k = kb * ORC_GROUP; k < (kb + 1) * ORC_GROUP; ++k) {\n"
                        "                    double prod = table[xr[k]] * fabs(table[wr[k]]);"),
    "rowcol_abs_weight": ("for (int64_t k = 0; k < K; ++k) {\n"
                          "                double prod = table[xr[k]] * table[wr[k]];",
                          "for (int64_t k = 0; k < K; ++k) {\n"
                          "                double prod = table[xr[k]] * fabs(table[wr[k]]);"),
    "grouped_segment_boundary": ("if (offs[i] <= m && m < offs[i + 1]) { e = i; break; }",
                                 "if (offs[i] <= m && m <= offs[i + 1]) { e = i; break; }"),
    "row_amax_half_row": ("float s = orc_scale_f32(amax_clamped(xr, K, 0, 1));",
                          "float s = orc_scale_f32(amax_clamped(xr, K / 2, 0, 1));"),
    "tensor_amax_first_row": ("return orc_scale_f32(amax_clamped(X, K, ldx, R));",
                              "return orc_scale_f32(amax_clamped(X, K, ldx, 1));"),
    "static_multiplies_by_scale": ("for (int64_t r = 0; r < R; ++r) quantize_run(X + r * ldx, K, s, Xq + r * K);",
                                   "for (int64_t r = 0; r < R; ++r) quantize_run(X + r * ldx, K, 1.0f / s, Xq + r * K);"),
    "rowcol_channel_scale_ignored": ("double c = a * (double)sw[w_per_tensor ? 0 : n];",
                                     "double c = a * (double)sw[0];"),
    "rowcol_token_scale_indexed_by_n": ("double a = (double)sx[x_per_tensor ? 0 : m];",
                                        "double a = (double)sx[x_per_tensor ? 0 : (m % 2)];"),
}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_c = tmp_path / "oracle_mutant.c"
    mutant_c.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                    "-w", "-o", str(so), str(mutant_c), "-lm"], check=True)
    env = dict(os.environ, FGFP8_ORACLE_LIB=str(so), OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_TESTS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
