"""The pins catch plausible mistakes in the oracle.

Each case copies oracle/nq_oracle.c, plants one mistake (a wrong sign, a
dropped term, a swapped index, a wrong tie rule, a wrong constant), builds
it, and runs the pin expected to catch it in a subprocess pointed at the
mutated library (NQ_ORACLE_SO).  The pin must fail; the unmutated oracle
passes the same pins in the rest of the suite.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nq_oracle.c")

# (id, original text, planted mistake, pin that must fail)
MUTATIONS = [
    ("fwht-butterfly-sign", "v[i + h] = a - b;", "v[i + h] = b - a;",
     "tests/test_oracle_transforms.py::test_fwht_equals_hadamard_matrix"),
    ("rope-undo-sign", "v[i + OQ_HALF] = fmaf(b, c[i], -as);", "v[i + OQ_HALF] = fmaf(b, c[i], as);",
     "tests/test_oracle_transforms.py::test_rope_undo_recovers_prerope_keys"),
    ("rope-table-combine", "c[i] = fmaf(ca, cb, -ss);", "c[i] = fmaf(ca, cb, ss);",
     "tests/test_oracle_transforms.py::test_rope_tables_vs_fp64"),
    ("e8-fix-direction", "f[k] += (e[k] >= 0.0f) ? 1 : -1;", "f[k] += (e[k] >= 0.0f) ? -1 : 1;",
     "tests/test_oracle_e8.py::test_optimal_vs_brute_force"),
    ("e8-dropped-fix-cost", "d = d + fmaf(-2.0f, m, 1.0f);", "d = d;",
     "tests/test_oracle_e8.py::test_optimal_vs_brute_force"),
    ("e8-coset-choice", "if (d1 < d0) {", "if (d1 > d0) {",
     "tests/test_oracle_e8.py::test_golden_examples"),
    ("scale-constant-swapped", "#define OQ_G3_BITS 0x3CCEE116u", "#define OQ_G3_BITS 0x3D715BEFu",
     "tests/test_oracle_codec.py::test_encode_matches_fp64_restatement"),
    ("clamp-range", "int32_t lim = (1 << bits) - (half ? 1 : 2);",
     "int32_t lim = (1 << bits) - (half ? 2 : 1);",
     "tests/test_oracle_e8.py::test_clamp_ranges"),
    ("pack-bit-index", "words[(bitpos + k) >> 5] |= 1u << ((bitpos + k) & 31);",
     "words[(bitpos + k) >> 5] |= 1u << ((bitpos + 2 - k) & 31);",
     "tests/test_oracle_codec.py::test_encode_matches_fp64_restatement"),
    ("decode-coset-offset", "int32_t t = 2 * (int32_t)j - (1 << bits) + 2 - h;",
     "int32_t t = 2 * (int32_t)j - (1 << bits) + 2 + h;",
     "tests/test_oracle_codec.py::test_decode_every_code_at_every_coordinate"),
    ("score-window-mean", "m[h * OQ_D + d] = (float)(S / (double)W);",
     "m[h * OQ_D + d] = (float)(S / (double)(W + 1));",
     "tests/test_oracle_select.py::test_score_matches_long_double"),
    ("select-tie-rule", "return (a->t > b->t) - (a->t < b->t);",
     "return (a->t < b->t) - (a->t > b->t);",
     "tests/test_oracle_select.py::test_select_ties_prefer_lower_position"),
    ("kept-count", "return T - (mid * pct) / 100;", "return T - (T * pct) / 100;",
     "tests/test_oracle_select.py::test_kept_count_rule"),
    ("attend-gqa-index", "const float *qj = q + (size_t)(h * G + g) * OQ_D;",
     "const float *qj = q + (size_t)(g * H + h) * OQ_D;",
     "tests/test_oracle_attend.py::test_attention_equals_library_softmax"),
    ("attend-lse", "lse[h * G + g] = m + log(l);", "lse[h * G + g] = log(l);",
     "tests/test_oracle_attend.py::test_attention_equals_library_softmax"),
    ("ans-table-tie", "if (F[s] > F[best]) best = s;", "if (F[s] >= F[best]) best = s;",
     "tests/test_oracle_entropy.py::test_table_rule_worked_examples"),
    ("ans-renorm-threshold", "if ((uint64_t)x >= ((uint64_t)f << 20)) {",
     "if ((uint64_t)x >= ((uint64_t)f << 21)) {",
     "tests/test_oracle_entropy.py::test_round_trip_and_size_bound"),
    ("ans-cumulative-offset", "x = (x / f) * OQ_ANS_M + (x % f) + C[s];",
     "x = (x / f) * OQ_ANS_M + (x % f) + C[s] + 1;",
     "tests/test_oracle_entropy.py::test_round_trip_and_size_bound"),
    ("entropy-delta-reference", "        prev = j;\n", "        prev = 0;\n",
     "tests/test_oracle_entropy.py::test_store_layout_matches_a_numpy_restatement"),
    ("box-move-direction", "if (f[i] + dir > hi || f[i] + dir < lo) dir = -dir;", ";",
     "tests/test_oracle_box.py::test_points_are_in_e8_and_in_the_box"),
    ("exact-unpack-parity", "par ^= j[i] & 1u;", "par ^= j[i] & 0u;",
     "tests/test_oracle_box.py::test_exact_packing_round_trip"),
]


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_planted_mistake(tmp_path, name, old, new, pin):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique or missing"
    mutated = tmp_path / "nq_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "liboq_mut.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(mutated), "-o", str(so), "-lm"])
    env = dict(os.environ, NQ_ORACLE_SO=str(so))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          pin], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"pin {pin} did not catch '{name}':\n{res.stdout[-1500:]}"
    assert "failed" in res.stdout or "error" in res.stdout.lower()
