"""Each plausible mistake planted in a copy of the oracle must fail a pin.

The copy is compiled on the CPU into a temporary directory and exercised in a
child process (a mistake that indexes out of bounds may crash it, which also
counts as caught); the real oracle is not touched."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(os.path.dirname(oracle.__file__), "si_oracle.c")

MUTANTS = {
    "drop_last_d": ("for (int d = 0; d < D; ++d) {", "for (int d = 0; d < D - 1; ++d) {"),
    "no_relu": ("double r = dot[h] > 0.0 ? dot[h] : 0.0;", "double r = dot[h];"),
    "relu_abs": ("double r = dot[h] > 0.0 ? dot[h] : 0.0;", "double r = dot[h] > 0.0 ? dot[h] : -dot[h];"),
    "weight_of_head0": ("wrow[h] = (double)p->w[base + h];", "wrow[h] = (double)p->w[base];"),
    "score_sign": ("acc += wrow[h] * r;", "acc -= wrow[h] * r;"),
    "visible_late": ("int64_t n = (t + 1) / m;", "int64_t n = t / m;"),
    "visible_early": ("int64_t n = (t + 1) / m;", "int64_t n = (t + m) / m;"),
    "no_T_cap": ("return n < T ? n : T;", "return n;"),
    "ties_high_index": ("return (a->idx > b->idx) - (a->idx < b->idx);",
                        "return (a->idx < b->idx) - (a->idx > b->idx);"),
    "ascending": ("if (a->score > b->score) return -1;\n  if (a->score < b->score) return 1;",
                  "if (a->score < b->score) return -1;\n  if (a->score > b->score) return 1;"),
    "pad_zero": ("out_idx[o] = -1;", "out_idx[o] = 0;"),
    "key_row_uses_S": ("int64_t r = b * p->T + s;", "int64_t r = b * p->S + s;"),
    "query_transposed": ("qrow[d * p->H + h] = oracle_bf16_value", "qrow[h * p->D + d] = oracle_bf16_value"),
    "e4m3_bias8": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "fp8_ignore_kscale": ("* (double)p->kc_scale[r];", ";"),
    "e2m1_bias2": ("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)"),
    "mx_nibbles_swapped": ("(d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15)",
                           "(d & 1) ? (uint8_t)(byte & 15) : (uint8_t)(byte >> 4)"),
    "mx_one_scale_per_row": ("scales[r * (D / 32) + d / 32]", "scales[r * (D / 32)]"),
    "e8m0_bias126": ("return ldexp(1.0, (int)bits - 127);", "return ldexp(1.0, (int)bits - 126);"),
    "pool_first_keys_only": ("for (int64_t i = 0; i < G; ++i) {\n      widen_key(p, b, j * G + i, krow);",
                             "for (int64_t i = 0; i < G - 1; ++i) {\n      widen_key(p, b, j * G + i, krow);"),
    "pool_no_bf16_rounding": ("= round_bf16(pool[j * p->D + d] / (double)G);", "= pool[j * p->D + d] / (double)G;"),
    "two_stage_no_tail": ("for (int64_t s = nbv * G; s < n; ++s) c[nc++].idx = s;", ""),
    "two_stage_keep_one_less": ("int64_t kept = nbv < n_keep ? nbv : n_keep;",
                                "int64_t kept = nbv < n_keep - 1 ? nbv : n_keep - 1;"),
    "two_stage_worst_blocks": ("c[nc++].idx = blk[j].idx * G + e;", "c[nc++].idx = blk[nbv - 1 - j].idx * G + e;"),
    "two_stage_incomplete_block": ("int64_t nbv = n / G;", "int64_t nbv = (n + G - 1) / G < nb ? (n + G - 1) / G : nb;"),
    "attn_no_scale": ("logit[j] = scale * dot;", "logit[j] = dot;"),
    "attn_value_from_tail": ("o[d] += e * oracle_bf16_value(vr[d]);", "o[d] += e * oracle_bf16_value(vr[Dk - Dv + d]);"),
    "attn_not_normalised": ("for (int64_t d = 0; d < Dv; ++d) o[d] /= den;", ""),
    "attn_padding_read": ("if (sel[j] < 0) continue;", "if (sel[j] < -1) continue;"),
}

RUNNER = r"""
import sys
sys.path.insert(0, sys.argv[1])
import oracle
from tests import oracle_pins
lib = oracle.load(sys.argv[2])
caught = []
for pin in oracle_pins.ALL:
    try:
        pin(lib)
    except Exception as e:
        caught.append(pin.__name__)
print("CAUGHT", ",".join(caught))
sys.exit(0 if caught else 3)
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(msrc), out=str(tmp_path / "libmutant.so"))
    r = subprocess.run([sys.executable, "-c", RUNNER, ROOT, so], capture_output=True, text=True,
                       timeout=300)
    # exit 0: some pin failed; negative: the mutant crashed the process
    assert r.returncode == 0 or r.returncode < 0, f"mutant {name} passed every pin\n{r.stdout}{r.stderr}"
