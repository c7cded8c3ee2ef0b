"""The oracle's pins must catch plausible mistakes.

Each case plants one bug in a copy of hils_oracle.c (on the CPU, in a
temporary directory), builds it, and runs the pin tests against that build:
at least one pin must fail.  The committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hils_oracle.c")

MUTATIONS = {
    "score_scale_dropped": ("return acc / sqrt((double)d);", "return acc;"),
    "attention_scale_dropped": ("logit[t - t0] = acc / sqrt((double)d);", "logit[t - t0] = acc;"),
    "attention_uses_calibrated_q": ("chunk_attention(c, q, ", "chunk_attention(c, qt, "),
    "scores_use_raw_q": ("ssel[a] = landmark_score(c, qt,", "ssel[a] = landmark_score(c, q,"),
    "scores_use_raw_q_all": ("s[j] = landmark_score(c, qt,", "s[j] = landmark_score(c, q,"),
    "tie_to_higher_index": ("if (best < 0 || s[j] > s[best]) best = j;",
                            "if (best < 0 || s[j] >= s[best]) best = j;"),
    "own_chunk_not_causal": ("if (t1 > pos) t1 = pos;", ""),
    "own_chunk_drops_last_key": ("int64_t t1 = t0 + S - 1;", "int64_t t1 = t0 + S - 2;"),
    "calibration_transposed_A": ("q[e] * (double)A[(int64_t)e * r + a]", "q[e] * (double)A[(int64_t)a * d + e]"),
    "calibration_sign": ("qt[e] = q[e] + acc;", "qt[e] = q[e] - acc;"),
    "uniform_fusion": ("w[a] = exp(ssel[a] - m) / z;", "w[a] = 1.0 / n;"),
    "gqa_modulo_mapping": ("return h / (c->n_q_heads / c->n_kv_heads);", "return h % c->n_kv_heads;"),
    "values_read_from_keys": ("kv_index(c, block_table, max_chunks, b, t, 1, g, e)",
                              "kv_index(c, block_table, max_chunks, b, t, 0, g, e)"),
    "softmax_max_not_subtracted_in_weights": ("z += exp(ssel[a] - m);", "z += exp(ssel[a]);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_bug(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = tmp_path / "hils_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", str(lib),
                           str(mutated), "-lm"])
    env = dict(os.environ, HILS_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"no pin caught mutation {name}:\n{r.stdout[-2000:]}"
