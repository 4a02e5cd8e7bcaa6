"""The oracle's pins catch plausible mistakes: each case plants one mistake in a
copy of oracle/salad_oracle.c (built in a temporary directory, on the CPU),
runs the pin files of that part of the oracle against the copy, and expects
them to fail.  The committed oracle is never changed; the unmutated pins run
in the rest of the CPU suite."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "salad_oracle.c")

MASK = ["tests/test_oracle_mask.py"]
FWD = ["tests/test_oracle_forward.py"]
GATE = ["tests/test_oracle_gate.py"]
BWD = ["tests/test_oracle_backward.py"]
TILE = ["tests/test_oracle_tiles.py"]
TOPK = ["tests/test_oracle_topk.py"]

# (name, text in the source, replacement, occurrences replaced, pin files)
MUTANTS = [
    ("mask: window one short in t", "for (int t2 = t - wt; t2 <= t + wt; ++t2)",
     "for (int t2 = t - wt; t2 < t + wt; ++t2)", 1, MASK),
    ("mask: x window ignored", "const int x_hi = x + ww > W - 1 ? W - 1 : x + ww;",
     "const int x_hi = x > W - 1 ? W - 1 : x;", 1, MASK),
    ("forward: no softmax scale", "s[t] = tau * dot;", "s[t] = dot;", 1, FWD),
    ("forward: S transposed", "u += pq * Sb[(int64_t)c * d + e];", "u += pq * Sb[(int64_t)e * d + c];", 1, FWD),
    ("forward: eps dropped", "lin[e] = u / (dn + eps);", "lin[e] = u / dn;", 1, FWD),
    ("forward: W transposed", "y += lin[c] * W[c * d + e];", "y += lin[c] * W[e * d + c];", 1, FWD),
    ("forward: gate dropped", "out[ooff + e] = acc[e] + g * y;", "out[ooff + e] = acc[e] + y;", 1, FWD),
    ("forward: relu of k dropped in the state", "pk[c] = kv > 0.0 ? kv : 0.0;", "pk[c] = kv;", 1, FWD),
    ("forward: relu of q dropped", "const double pq = qi[c] > 0.0 ? qi[c] : 0.0;", "const double pq = qi[c];", 2, FWD),
    ("forward: softmax not normalised", "acc[c] /= den;", "acc[c] /= 1.0;", 1, FWD),
    ("forward: last kept block of a row skipped",
     "for (int32_t r = r0; r < r1; ++r) {\n            block_tokens(geom, N, blk, col_idx[r], slot_tok);",
     "for (int32_t r = r0; r < r1 - 1; ++r) {\n            block_tokens(geom, N, blk, col_idx[r], slot_tok);", 1, FWD),
    ("gate: sum for mean", "logit += w_x[(size_t)h * d + f] * (sum / N);",
     "logit += w_x[(size_t)h * d + f] * sum;", 1, GATE),
    ("gate: sigmoid sign", "1.0 / (1.0 + exp(-logit))", "1.0 / (1.0 + exp(logit))", 1, GATE),
    ("gate: drops at the threshold", "sv < threshold ? 0.0 : sv", "sv <= threshold ? 0.0 : sv", 1, GATE),
    ("backward: D_i dropped", "const double ds = sc[t] * (dp - D);", "const double ds = sc[t] * dp;", 1, BWD),
    ("backward: dW transposed", "+= orow[ri * d + e] * g * dout[off + f];",
     "+= orow[ri * d + f] * g * dout[off + e];", 1, BWD),
    ("backward: dden sign", "dden[ri] = -od / den;", "dden[ri] = od / den;", 1, BWD),
    ("backward: dv from ds", "av[c] += p * dout[qoff + c];", "av[c] += ds * dout[qoff + c];", 1, BWD),
    ("backward: dgate from o", "ygi += gi[f] * y[f];", "ygi += gi[f] * o[f];", 1, BWD),
    ("tiles: y window one short", "llabs(y - y2) <= wh && llabs(x - x2) <= ww",
     "llabs(y - y2) < wh && llabs(x - x2) <= ww", 1, TILE),
    ("tiles: boxes numbered column-major", "xi = (int)(I % nw);", "xi = (int)((I / nh) % nw);", 1, TILE),
    ("topk: keeps the lowest scores", "if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
     "if (x->score < y->score) return -1;\n    if (x->score > y->score) return 1;", 1, TOPK),
    ("topk: ties keep the larger block", "return (x->j > y->j) - (x->j < y->j);",
     "return (x->j < y->j) - (x->j > y->j);", 1, TOPK),
    # (on the key side: the query mean of a row scales all of that row's scores
    # alike, so the same mistake there leaves the ranking unchanged)
    ("topk: partial key block averaged over the block size", "km[(int64_t)I * d + c] = sk / (float)(t1 - t0);",
     "km[(int64_t)I * d + c] = sk / (float)blk;", 1, TOPK),
    ("lse: running maximum left out", "l > 0.0 ? m + log(l) : -INFINITY;", "l > 0.0 ? log(l) : -INFINITY;", 1, BWD),
    ("backward: relu derivative dropped in dq", "if (!(qi[c] > 0.0)) continue;", "if (0) continue;", 1, BWD),
    ("backward: dk without the relu mask", "if (kj[c] > 0.0) {", "if (1) {", 1, BWD),
    ("backward: dz left out of dk", "double t = dzb[c];", "double t = 0.0;", 1, BWD),
]


@pytest.mark.parametrize("name,old,new,count,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, count, pins):
    src = open(SRC).read()
    assert src.count(old) == count, f"mutation site not found: {name}"
    mutant = tmp_path / "salad_oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libsalad_oracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(lib), str(mutant),
                           "-lm"])
    env = dict(os.environ, SALAD_ORACLE_LIB=str(lib))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                          *pins], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"{name}: the pins passed with the mistake planted\n{res.stdout[-2000:]}"
    # a pin failed (an assertion), as opposed to a crash of the run
    assert " failed" in res.stdout, f"{name}: the run ended without a failed pin\n{res.stdout[-2000:]}"


def test_pins_pass_on_an_unmutated_copy(tmp_path):
    """The control: the same build of the unchanged source passes every pin file
    used above, so a failure above is the planted mistake's."""
    lib = tmp_path / "libsalad_oracle_copy.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(lib), SRC, "-lm"])
    env = dict(os.environ, SALAD_ORACLE_LIB=str(lib))
    pins = sorted({f for m in MUTANTS for f in m[4]})
    res = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu", *pins],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:]
