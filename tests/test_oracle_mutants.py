"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (a dropped term, a wrong
sign or index, a transposed operand, a different rounding rule), builds it on
the CPU, and runs the pin suites against that copy in a subprocess: the suites
must fail.  The oracle itself is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "rmsnorm_no_eps": ("ss / (double)n + RMS_EPS", "ss / (double)n"),
    "rmsnorm_sum_not_mean": ("sqrt(ss / (double)n + RMS_EPS)", "sqrt(ss + RMS_EPS)"),
    "matvec_transposed": ("v += (double)row[j] * (double)x[j];", "v += (double)W[(size_t)j * d + i] * (double)x[j];"),
    "rope_sign": ("v[i] = (float)(a * c - b * s);", "v[i] = (float)(a * c + b * s);"),
    "rope_freq_index": ("orc_rope_freq(i % head_size, head_size)", "orc_rope_freq(i, head_size)"),
    "attn_no_scale": ("att[t] = s * scale;", "att[t] = s;"),
    "gqa_mapping": ("int g = h / rep;", "int g = h % n_kv_heads;"),
    "silu_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "quant_round_half_even": ("q[g * gs + i] = (int8_t)round((double)quot);", "q[g * gs + i] = (int8_t)rint((double)quot);"),
    "quant_scale_128": ("return orc_quantize_qmax(x, n, gs, 127.0f, q, s);", "return orc_quantize_qmax(x, n, gs, 128.0f, q, s);"),
    "q4_scale_8": ("return orc_quantize_qmax(x, n, gs, 7.0f, q, s);", "return orc_quantize_qmax(x, n, gs, 8.0f, q, s);"),
    "q4_set_holds_q8_codes": ("return four ? orc_quantize4(", "return 0 ? orc_quantize4("),
    "q4_embedding_row_from_fp32": ("    if (z) orc_dequantize(z->E.q + (size_t)token * d, z->E.s + (size_t)token * d / z->gs, d, z->gs, x);\n    else memcpy(",
                                   "    if (z && z == &m->q8) orc_dequantize(m->q8.E.q + (size_t)token * d, m->q8.E.s + (size_t)token * d / m->q8.gs, d, m->q8.gs, x);\n    else memcpy("),
    "q80_drop_sx": ("vd += (double)ival * (double)srow[g] * (double)sx[g];", "vd += (double)ival * (double)srow[g];"),
    "no_attn_residual": ("for (int i = 0; i < d; i++) x[i] += m->xb2[i];", "for (int i = 0; i < d; i++) x[i] = m->xb2[i];"),
    "no_rope_on_k": ("orc_rope(k, kvd, hs, pos);", ""),
    "argmax_last_tie": ("if (x[i] > x[best]) best = i;", "if (x[i] >= x[best]) best = i;"),
    "wrong_norm_weight": ("orc_rmsnorm(m->xb, x, m->w_att + l * d, d);", "orc_rmsnorm(m->xb, x, m->w_ffn + l * d, d);"),
    "kv8_before_rope": ("        orc_rope(k, kvd, hs, pos);\n        if (m->kv8) {\n            orc_kv8_row(k, kvd, hs);",
                        "        if (m->kv8) orc_kv8_row(k, kvd, hs);\n        orc_rope(k, kvd, hs, pos);\n        if (m->kv8) {"),
    "kv8_v_not_quantized": ("            orc_kv8_row(v, kvd, hs);\n        }", "        }"),
    "kv8_one_group_per_row": ("            orc_kv8_row(k, kvd, hs);\n", "            orc_kv8_row(k, kvd, kvd);\n"),
    "swiglu_operands_swapped": ("orc_swiglu(m->hb, m->hb2, h);", "orc_swiglu(m->hb2, m->hb, h); memcpy(m->hb, m->hb2, sizeof(float) * (size_t)h);"),
    "sample_temperature_multiplies": ("((double)z[i] - (double)mx) / (double)temperature", "((double)z[i] - (double)mx) * (double)temperature"),
    "sample_topp_excludes_ties": ("for (int i = 0; i < n; i++) if (q[i] >= tau) zset += q[i];", "for (int i = 0; i < n; i++) if (q[i] > tau || (q[i] == tau && i == 0)) zset += q[i];"),
    "sample_coin_not_scaled": ("const double target = coin * zset;", "const double target = coin;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    find, repl = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(find) == 1, f"mutation anchor not found once: {find}"
    with tempfile.TemporaryDirectory() as td:
        msrc = os.path.join(td, "oracle.c")
        with open(msrc, "w") as f:
            f.write(src.replace(find, repl))
        with open(os.path.join(td, "oracle.h"), "w") as f:
            f.write(open(os.path.join(ROOT, "oracle", "oracle.h")).read())
        so = os.path.join(td, "liboracle_mutant.so")
        subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", so, msrc, "-lm"])
        env = dict(os.environ, ORACLE_LIB_PATH=so, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            "tests/test_oracle_pins.py", "tests/test_oracle_forward.py",
                            "tests/test_oracle_sampling.py", "tests/test_oracle_kv8.py"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
