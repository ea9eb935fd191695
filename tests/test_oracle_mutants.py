"""The oracle's pins must catch plausible mistakes.  Each case plants one mistake in a
temporary copy of the oracle's C source (a dropped term, a wrong sign or index, a transposed
operand, a wrong tie-break, a missing rounding), builds it, runs the pin tests of
tests/test_oracle.py against that build, and requires at least one of them to fail.  The
committed oracle is never modified."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

# (name, text in the source, planted replacement)
MUTANTS = [
    ("router_transposed_Wg", "l[i] += xj * (double)Wg[j * n + i];",
     "l[i] += xj * (double)Wg[i * d + j];"),
    ("tie_break_higher_index", "(l[a] == l[b] && a < b)", "(l[a] == l[b] && a > b)"),
    ("softmax_not_shifted_normalised", "gate[k] = exp(l[order[k]] - top) / z;",
     "gate[k] = exp(l[order[k]] - top);"),
    ("gate_uses_wrong_slot", "gate[k] = exp(l[order[k]] - top) / z;",
     "gate[k] = exp(l[order[K - 1 - k]] - top) / z;"),
    ("w1_w3_swapped", "double hf = oracle_silu(a) * b;", "double hf = oracle_silu(b) * a;"),
    ("silu_dropped", "double hf = oracle_silu(a) * b;", "double hf = a * b;"),
    ("w3_term_dropped", "b += xt[j] * elem(W3, w_dtype, w13 + f * d + j);", "b += 0.0;"),
    ("w2_transposed", "yi += h[f] * elem(W2, w_dtype, w2 + i * F + f);",
     "yi += h[f] * elem(W2, w_dtype, w2 + (f % d) * F + (i % F));"),
    ("gate_weight_dropped", "acc[i] += g * yi;", "acc[i] += yi;"),
    ("h_not_rounded", "h[f] = h_dtype < 0 ? hf : round_to(hf, h_dtype);", "h[f] = hf;"),
    ("bf16_one_bit_short", "int q = e - 8;", "int q = e - 7;"),
    ("rmsnorm_eps_dropped", "1.0 / sqrt(ss / (double)d + eps);", "1.0 / sqrt(ss / (double)d);"),
    ("residual_dropped", "round_to(x[r * d + i] + yr[i], dtype);", "round_to(yr[i], dtype);"),
    ("e4m3_ties_to_odd", "(dist == bd && (c & 1) == 0)", "(dist == bd && (c & 1) == 1)"),
    ("mx_exponent_off_by_one", "int E = f <= 0.875 ? ex - 9 : ex - 8;",
     "int E = f <= 0.875 ? ex - 8 : ex - 7;"),
    ("mx_clipping_rule", "int E = f <= 0.875 ? ex - 9 : ex - 8;", "int E = ex - 9;"),
    ("mx_threshold_at_one_and_a_half", "int E = f <= 0.875 ? ex - 9 : ex - 8;",
     "int E = f <= 0.75 ? ex - 9 : ex - 8;"),
    ("mx_low_clamp_dropped", "if (E < -127) E = -127;", "if (E < -200) E = -127;"),
    ("mx_zero_block_scale", "if (amax == 0.0f) return 127;", "if (amax == 0.0f) return 0;"),
    ("mx_overflow_to_nan", "if (a >= 448.0) return sign | 126;", "if (a > 464.0) return sign | 127;"),
    ("e4m3_subnormal_step", "ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    ("fp8_activation_scale_dropped",
     "total += oracle_e8m0_value(sa[b]) * oracle_e8m0_value(sw[b]) * s;",
     "total += oracle_e8m0_value(sw[b]) * s;"),
    ("fp8_w3_uses_w1",
     "const double b = mx_dot(qx, sx, W3q + wr * d, sf3 + wr * bd, d, lut);",
     "const double b = mx_dot(qx, sx, W1q + wr * d, sf1 + wr * bd, d, lut);"),
    ("fp8_h_block_scales_shifted", "mx_quantize_row(hf, F, qh, sh);",
     "mx_quantize_row(hf, F, qh, sh); sh[0] = sh[bf - 1];"),
]


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, source, name, old, new):
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    mdir = tmp_path / "oracle"
    mdir.mkdir()
    (mdir / "moe_oracle.c").write_text(source.replace(old, new))
    with open(os.path.join(ROOT, "oracle", "__init__.py")) as f:
        (mdir / "__init__.py").write_text(f.read())
    env = dict(os.environ, MOE_ORACLE_MUTANT_DIR=str(tmp_path))
    # the pins, run against the mutant build (its own package dir shadows the real oracle)
    proc = subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
         os.path.join(HERE, "test_oracle.py"), "--rootdir", str(tmp_path),
         "-c", os.path.join(ROOT, "pytest.ini")],
        cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=600)
    assert proc.returncode != 0, f"mutant {name} survived the pins:\n{proc.stdout[-2000:]}"
    assert "failed" in proc.stdout, proc.stdout[-2000:]
    assert os.path.exists(mdir / "libmoe_oracle.so"), "the mutant build was not the one tested"
