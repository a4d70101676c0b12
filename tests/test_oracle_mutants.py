"""Mutation check of the oracle pins (CPU only).

Each case plants one plausible mistake in a copy of the oracle's C source (a wrong constant,
a dropped term, a transposed operand, a wrong tie rule, a swapped nibble), builds it, and
runs the pin suite against it in a subprocess: the suite must reject every mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nvfp4_oracle.c")

MUTANTS = {
    "fp8_max_448_in_four_over_six": ('nvo_quantize_ex(x, groups, rows, cols, amax, 256.0f, 3,',
                                     'nvo_quantize_ex(x, groups, rows, cols, amax, 448.0f, 3,'),
    "six_m_uses_4": ("float six_m = 6.0f * fp8_max;", "float six_m = 4.0f * fp8_max;"),
    "e2m1_step_1_above_2_kept_to_4": ("(a < 4.0 ? 1.0 : 2.0)", "(a < 6.0 ? 1.0 : 2.0)"),
    "e2m1_ties_away": ("v = rint(a / step) * step;\n        if (v > 6.0)",
                       "v = floor(a / step + 0.5) * step;\n        if (v > 6.0)"),
    "e4m3_truncates": ("v = rint(a / step) * step;        /* a/step is exact",
                       "v = floor(a / step) * step;        /* a/step is exact"),
    "mse_drops_odd_terms": ("default:              acc[i & 1] = fmaf(c->e[i], c->e[i], acc[i & 1]); break;",
                            "default:              if (!(i & 1)) acc[0] = fmaf(c->e[i], c->e[i], acc[0]); break;"),
    "mae_uses_squares": ("case NVO_RULE_MAE:    acc[i & 1] = acc[i & 1] + ae; break;",
                         "case NVO_RULE_MAE:    acc[i & 1] = acc[i & 1] + ae * ae; break;"),
    "choice_prefers_4_on_ties": ("four = (c4.err < c6.err);", "four = (c4.err <= c6.err);"),
    "choice_inverted": ("four = (c4.err < c6.err);", "four = (c4.err > c6.err);"),
    "nibbles_swapped": ("(uint8_t)(chosen->code[2 * j] | (chosen->code[2 * j + 1] << 4))",
                        "(uint8_t)(chosen->code[2 * j + 1] | (chosen->code[2 * j] << 4))"),
    "decode_scale_transposed": ("c->d = nvo_e4m3_to_f32(c->s) * alpha;", "c->d = nvo_e4m3_to_f32(c->s) / alpha;"),
    "error_against_scaled_values": ("c->e[i] = fmaf(-v, c->d, x[i]);", "c->e[i] = y - v;"),
    "error_drops_scale": ("c->e[i] = fmaf(-v, c->d, x[i]);", "c->e[i] = x[i] - v;"),
    # the other reading of the error term: the dequantized value rounded before the subtraction
    "error_rounds_product_first": ("c->e[i] = fmaf(-v, c->d, x[i]);", "c->e[i] = x[i] - c->q[i];"),
    "zero_sign_dropped": ("uint8_t sign = signbit(y) ? 0x8u : 0x0u;", "uint8_t sign = (y < 0) ? 0x8u : 0x0u;"),
    "kl_reversed": ("acc += p * (logp - logq);", "acc += q * (logq - logp);"),
    "kl_grad_sign": ("grad[r * vocab + v] = grad_scale * (q - p);", "grad[r * vocab + v] = grad_scale * (p - q);"),
    "kl_student_normalizer_dropped": ("double logp = a - lse_t, logq = b - lse_s;", "double logp = a - lse_t, logq = b - ms;"),
    "kl_tau_on_teacher_only": ("zs += exp(nvo_bf16_to_f32(s[v]) / tau - ms);", "zs += exp(nvo_bf16_to_f32(s[v]) - ms);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    mut = tmp_path / "nvfp4_oracle.c"
    mut.write_text(src.replace(old, new))
    hdr = os.path.join(ROOT, "oracle")
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
                    "-I", hdr, str(mut), "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, NVO_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_qad_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins accepted mutant {name}:\n{r.stdout[-2000:]}"
