"""Plant plausible mistakes in a copy of the oracle and check the pins catch them.

Each mutant is rat_oracle.c with one textual change (a swapped gate, a wrong
sign, a dropped term, a wrong dilation residue, a window off by one, a wrong
merge, a dropped scale, a transposed operand, a gate one step late, a decode
that ignores the per-head recurrence flag, a fixed grid on the wrong residue
or without the query's own key, a dedupe that keeps the shared keys,
a top-k block selection with a one-sided bound, a dropped first or local
block, ties to the wrong block, one block too many or a selection gap of
the wrong sign).  It is compiled into a temporary
directory and the pin suite is run against it in a subprocess; the suite must
fail.  The shipped oracle is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rat_oracle.c")

MUTANTS = {
    "gate_swapped": ("s = a * s + (1.0 - a) * x[e];", "s = (1.0 - a) * s + a * x[e];"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    "init_dropped": ("double s = init ? init[ch] : 0.0;", "double s = 0.0;"),
    "gate_one_step_late": ("double a = rec ? sigmoid(g[e]) : 0.0;",
                           "double a = rec ? sigmoid(g[t > 0 ? e - (size_t)H * d : e]) : 0.0;"),
    "residue_fixed_grid": ("if ((t - j) % D == 0) js[n++] = j;", "if (j % D == 0 || j == t) js[n++] = j;"),
    "window_off_by_one": ("if (j >= t - W + 1) js[n++] = j;", "if (j >= t - W) js[n++] = j;"),
    "merge_plain_average": ("o[c] = (w1 * o1[c] + w2 * o2[c]) / (w1 + w2);", "o[c] = 0.5 * (o1[c] + o2[c]);"),
    "merge_lse_dropped": ("*lse = m + log(w1 + w2);", "*lse = m;"),
    "scale_dropped": ("z[i] = scale * acc;", "z[i] = acc;"),
    "keys_read_values": ("acc += qrow[c] * k[idx4(T, H, d, b, js[i], h, c)];",
                         "acc += qrow[c] * v[idx4(T, H, d, b, js[i], h, c)];"),
    "decode_ignores_recur": ("double a = (recur == NULL || recur[h]) ? sigmoid(g[e]) : 0.0;",
                             "double a = sigmoid(g[e]);"),
    "grid_on_residue_zero": ("if (j % D == D - 1 || j == t) js[n++] = j;", "if (j % D == 0 || j == t) js[n++] = j;"),
    "grid_without_self": ("if (j % D == D - 1 || j == t) js[n++] = j;", "if (j % D == D - 1) js[n++] = j;"),
    "dedupe_ignored": ("if (!in_dil) js[n2++] = j;", "js[n2++] = j;"),
    "topk_quest_upper_end_only": ("sc += a1 > a2 ? a1 : a2;", "sc += a2;"),
    "topk_local_block_dropped": ("keep[blk] = (blk == 0 || blk == c);", "keep[blk] = (blk == 0);"),
    "topk_first_block_dropped": ("keep[blk] = (blk == 0 || blk == c);", "keep[blk] = (blk == c);"),
    "topk_ties_to_higher_block": ("(best < 0 || score[blk] > score[best])", "(best < 0 || score[blk] >= score[best])"),
    "topk_one_block_too_many": ("for (int pick = 0; pick < K; ++pick)", "for (int pick = 0; pick <= K; ++pick)"),
    "topk_gap_sign": ("last - rest;", "rest - last;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site not found: " + name
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(lib), str(msrc), "-lm"])
    env = dict(os.environ, RAT_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "mutant %s survived the pins:\n%s" % (name, r.stdout[-2000:])
