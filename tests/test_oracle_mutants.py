"""The oracle's pins catch planted mistakes.

Each mutant is oracle.c with one plausible mistake written in (a dropped or
transposed term, a wrong index, sign, weight, divisor or rule), compiled on
the CPU into a temporary library; the pin suite (test_oracle_pins.py, minus
the golden regression record, which the oracle itself wrote) runs against it
in a subprocess and must fail.  The oracle's own source is never modified.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, original text, mistaken text); each original occurs exactly once
MUTANTS = [
    ("slash_pooled_like_vertical", "shat[(p - j) / b] += a;", "shat[j / b] += a;"),
    ("vs_score_operands_swapped", "w[c] = vhat[c] + shat[r - c];", "w[c] = vhat[r - c] + shat[c];"),
    ("stats_divided_by_b_not_rows", "vhat[c] /= rows; shat[c] /= rows;", "vhat[c] /= rows; shat[c] /= b;"),
    ("jsd_second_weight_dropped", "return 0.5 * a + 0.5 * c;", "return 0.5 * a + c;"),
    ("nibble_high_term_wrong_power", "aH * bH * 256", "aH * bH * 128"),
    ("pattern_rule_inverted", "(*jsd < tau) ? ORC_QA : ORC_VS", "(*jsd < tau) ? ORC_VS : ORC_QA"),
    ("ties_by_higher_index", "return a < b ? -1 : (a > b ? 1 : 0);", "return a < b ? 1 : (a > b ? -1 : 0);"),
    ("gamma_stops_one_block_early", "if (cum >= gamma) break;", "if (cum + w[order[t]] >= gamma) break;"),
    ("diagonal_not_forced", "keep[r] = 1;", "keep[r] = 0;"),
    ("logit_scale_without_sqrt", "double inv = 1.0 / sqrt((double)P->d);", "double inv = 1.0 / (double)P->d;"),
    ("block_means_over_b_not_rows", "out[(size_t)c * d + t] = acc / cnt;", "out[(size_t)c * d + t] = acc / b;"),
    ("attention_mask_excludes_diagonal", "if (j <= p) { js[m] = j;", "if (j < p || p == 0) { js[m] = j;"),
    ("rope_rotation_sign", "orow[i] = round_bf16(xr[i] * c - xr[i + half] * sn);",
     "orow[i] = round_bf16(xr[i] * c + xr[i + half] * sn);"),
    ("rope_second_half_sign", "orow[i + half] = round_bf16(xr[i + half] * c + xr[i] * sn);",
     "orow[i + half] = round_bf16(xr[i + half] * c - xr[i] * sn);"),
    ("qa_softmax_without_max_shift", "for (int c = 0; c < m; ++c) { out[c] = exp(out[c] - mx); z += out[c]; }",
     "for (int c = 0; c < m; ++c) { out[c] = exp(out[c]); z += out[c]; }"),
    ("qa_logit_transposed", "acc += qbar[t] * kbar[(size_t)c * d + t];", "acc += qbar[c] * kbar[(size_t)t * d + c];"),
    # wiring of the whole-head index (which operand feeds which step)
    ("pest_from_first_block_qbar", "orc_pest(qbar + (size_t)(n - 1) * d, kbar, n, d, pest);",
     "orc_pest(qbar, kbar, n, d, pest);"),
    ("qa_rows_use_last_block_qbar", "orc_row_scores(*pattern, r, vhat, shat, qbar + (size_t)r * d, kbar, d, w);",
     "orc_row_scores(*pattern, r, vhat, shat, qbar + (size_t)(n - 1) * d, kbar, d, w);"),
    ("jsd_on_slash_not_vertical", "*jsd = orc_jsd(vhat, pest, n);", "*jsd = orc_jsd(shat, pest, n);"),
    ("kbar_of_wrong_kv_head", "int b = P->b, d = P->d, n = nblocks(P), kvh = h / (P->Hq / P->Hkv);",
     "int b = P->b, d = P->d, n = nblocks(P), kvh = h % P->Hkv;"),
    ("qbar_of_kv_head_index", "orc_block_means(P, 0, h, qbar);", "orc_block_means(P, 0, kvh, qbar);"),
    # head-pattern sharing and the block-size rule
    ("share_joins_any_earlier_head", "            if (cls[b] != b) continue;\n", ""),
    ("union_skips_last_member", "for (int m = 0; m < members; ++m)", "for (int m = 0; m + 1 < members; ++m)"),
    ("cover_count_one_short", "while (k < n && cum < gamma) cum += v[order[k++]];",
     "while (k + 1 < n && cum + v[order[k]] < gamma) cum += v[order[k++]];"),
    ("block_size_regimes_swapped", "if (rho >= 0.5) return 256;", "if (rho >= 0.5) return 64;"),
]


def build_mutant(tmp, name, orig, bad):
    src = open(SRC).read()
    assert src.count(orig) == 1, (name, src.count(orig))
    path_c = os.path.join(tmp, f"{name}.c")
    open(path_c, "w").write(src.replace(orig, bad))
    path_so = os.path.join(tmp, f"{name}.so")
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=gnu99", "-shared", "-fPIC",
                           path_c, "-o", path_so, "-lm"])
    return path_so


def run_pins(lib_path):
    env = dict(os.environ, ORACLE_LIB=lib_path)
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-x", "-q",
           "-p", "no:cacheprovider", "--deselect",
           "tests/test_oracle_pins.py::test_golden_tiny_index_regression"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def test_every_mutant_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        libs = [(name, build_mutant(tmp, name, orig, bad)) for name, orig, bad in MUTANTS]
        with ThreadPoolExecutor(4) as ex:
            results = list(ex.map(lambda nl: (nl[0],) + run_pins(nl[1]), libs))
    survivors = [name for name, rc, _ in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"


def test_unmutated_oracle_passes_the_same_run():
    """The same subprocess run on the real oracle passes (the harness itself works)."""
    from oracle import oracle as orc
    rc, out = run_pins(orc.build())
    assert rc == 0, out
