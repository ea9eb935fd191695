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
    ("e4m3_wrong_max", "return amax > 0.0f ? amax / 448.0f : 1.0f;",
     "return amax > 0.0f ? amax / 240.0f : 1.0f;"),
    ("e4m3_subnormal_step", "ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    ("fp8_x_scale_dropped", "const double a = (double)sx * (double)s1[(int64_t)e * F + f] * sa;",
     "const double a = (double)s1[(int64_t)e * F + f] * sa;"),
    ("fp8_h_scale_dropped",
     "yr[i] += gate[k] * ((double)sh * (double)s2[(int64_t)e * d + i] * sy);",
     "yr[i] += gate[k] * ((double)s2[(int64_t)e * d + i] * sy);"),
    ("fp8_w3_uses_w1", "sb += lut[qx[j]] * lut[w3[j]];", "sb += lut[qx[j]] * lut[w1[j]];"),
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
