"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Every mutant is a textual edit of ``oracle/retnet_oracle.c`` compiled into a scratch
library; the pin suite (``test_oracle_pins.py``) then runs in a subprocess against it
and must fail.  This is what makes the pins trustworthy: a dropped term, a wrong
exponent, sign or index, or a wrong variance would not slip through.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "retnet_oracle.c")

# (name, text in the oracle, replacement, occurrence index or None for all)
MUTANTS = [
    ("xi_exponent_r", "double xi = pow(g, (double)(r + 1));", "double xi = pow(g, (double)(r));", None),
    ("zeta_exponent", "pow(g, (double)(bl - 1 - r))", "pow(g, (double)(bl - r))", None),
    ("tail_decay_uses_B", "double gb = pow(g, (double)bl);", "double gb = pow(g, (double)chunk);", None),
    ("rotation_sign", "y[2 * j] = x0 * c - x1 * s;", "y[2 * j] = x0 * c + x1 * s;", None),
    ("key_turned_backwards",
     "xpos_rotate(row_qk(k, &d, b, t, hh), kr + t * d.d_k, d.d_k, theta, pos0 + t, xpos);",
     "xpos_rotate(row_qk(k, &d, b, t, hh), kr + t * d.d_k, d.d_k, theta, -(pos0 + t), xpos);", None),
    ("mask_drops_diagonal", "for (int64_t m = 0; m <= n; ++m)", "for (int64_t m = 0; m < n; ++m)", None),
    ("norm_r_without_abs", "fmax(fabs(sigma), 1.0)", "fmax(sigma, 1.0)", None),
    ("norm_d_row_sum_short", "for (int64_t j = 0; j <= p; ++j) rs +=", "for (int64_t j = 0; j < p; ++j) rs +=", None),
    ("recurrent_decay_on_input", "S[i * d.d_v + j] = g * S[i * d.d_v + j] + kn[i] * vn[j];",
     "S[i * d.d_v + j] = S[i * d.d_v + j] + g * kn[i] * vn[j];", None),
    ("sqrt_d_missing_root", "if (flags & ORACLE_F_SCALE_SQRT_D) f /= sqrt((double)d_k);",
     "if (flags & ORACLE_F_SCALE_SQRT_D) f /= (double)d_k;", None),
    ("groupnorm_unbiased", "var /= (double)d_v;", "var /= (double)(d_v - 1);", None),
    ("gate_sigmoid_not_swish", "double sw = gr[j] / (1.0 + exp(-gr[j]));",
     "double sw = 1.0 / (1.0 + exp(-gr[j]));", None),
    ("chunk_cross_term_dropped", "acc[j] += xi * cr;", "acc[j] += 0.0 * xi * cr;", None),
    ("state_in_ignored", "if (state_in) memcpy(S, state_in + bh * ssz", "if (0) memcpy(S, state_in + bh * ssz", None),
    ("bwd_state_term_dropped", "tq[i] += gn * dot(S0 + i * dv_, don, dv_);",
     "tq[i] += 0.0 * gn * dot(S0 + i * dv_, don, dv_);", None),
    ("bwd_rotation_not_transposed", "x[2 * j] = y0 * c + y1 * s;", "x[2 * j] = y0 * c - y1 * s;", None),
    ("bwd_dk_dv_without_row_factor", "double a = f[n] * pow(g, (double)(n - m));",
     "double a = pow(g, (double)(n - m));", None),
    ("bwd_dstate_decay_off_by_one", "double a = f[n] * pow(g, (double)(n + 1));",
     "double a = f[n] * pow(g, (double)n);", None),
]


@pytest.mark.parametrize("name,old,new,_", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new, _):
    src = open(SRC).read()
    assert old in src, f"mutation site for {name} not found; update the mutant table"
    mutant = src.replace(old, new)
    csrc = tmp_path / "mutant.c"
    csrc.write_text(mutant)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(csrc), "-o", str(lib),
                    "-lm"], check=True)
    env = dict(os.environ, RETNET_ORACLE_LIB_OVERRIDE=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
