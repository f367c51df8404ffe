"""Each plausible mistake in the oracle must fail at least one pin.

A mutation is planted in a temporary copy of oracle/csa_oracle.c (CPU only),
built with gcc, loaded in place of the real oracle (which is never touched),
and the pin suite is run against it; the test passes when some pin fails.
The mutants run several at a time, each in its own process.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "csa_oracle.c")

# (name, exact text in csa_oracle.c, replacement)
MUTATIONS = [
    ("b-window from block i instead of i-1", "int64_t tb = m * (i - 1) + r;", "int64_t tb = m * i + r;"),
    ("bias rows of the b-window swapped with the a-window",
     "bias[(m + r) * c + j]; /* Z^b + B^b */", "bias[r * c + j]; /* Z^b + B^b */"),
    ("Z^a used for the b-window logits", "rb[3 * c + j] + bias", "rb[2 * c + j] + bias"),
    ("C^a used for the b-window values", "acc += s * rb[1 * c + j];", "acc += s * rb[0 * c + j];"),
    ("block 0 b-window zero-padded instead of absent",
     "int has_b = (tb >= 0) || (left != NULL);", "int has_b = 1; if (tb < 0 && !left) { present[m + r] = 1; logit[m + r] = bias[(m + r) * c + j]; continue; }"),
    ("HCA bias ignored", "+ bias[r * c + j];   /* Z + B' */", ";   /* Z + B' */"),
    ("HCA values taken from Z", "acc += s * proj[(i * mp + r) * 2 * c + j];",
     "acc += s * proj[(i * mp + r) * 2 * c + c + j];"),
    ("HCA window shifted by one token", "logit[r] = proj[(i * mp + r) * 2 * c + c + j]",
     "logit[r] = proj[((i * mp + r + 1) % n) * 2 * c + c + j]"),
    ("indexer without ReLU", "(dot > 0.0 ? dot : 0.0)", "dot"),
    ("indexer sees its own block", "if (s >= vis) {", "if (s > vis) {"),
    ("indexer weight of head 0 for all heads", "acc += w[(int64_t)t * HI + h] *", "acc += w[(int64_t)t * HI] *"),
    ("top-k ties to the higher index", "return a < b;", "return a > b;"),
    ("top-k ascending", "return row[a] > row[b];", "return row[a] < row[b];"),
    ("MQA without scale", "z[i] = scale * dot;", "z[i] = dot;"),
    ("sink added to the numerator set twice", "if (sink) den += exp(sink[h] - mx);",
     "if (sink) den += 2.0 * exp(sink[h] - mx);"),
    ("dense MQA sees its own block", "int64_t vis = pos[t] / mp;", "int64_t vis = pos[t] / mp + 1;"),
    ("bf16 rounding truncates", "double r = ldexp(round_half_even(ldexp(a, -q)), q);\n    /* largest finite bf16",
     "double r = ldexp(floor(ldexp(a, -q)), q);\n    /* largest finite bf16"),
    ("projection loops use a transposed W index", "X[t * d + k] * W[o * d + k]",
     "X[t * d + k] * W[(k * M + o) % (M * d)]"),
    ("RMSNorm over the sum of squares instead of the mean", "sqrt(ss / c + eps)", "sqrt(ss + eps)"),
    ("rotary frequencies base^(-i/R)", "pow(base, -2.0 * i / R)", "pow(base, -1.0 * i / R)"),
    ("rotation turns the other way", "yr[j] = a * cos(ang) - b * sin(ang);", "yr[j] = a * cos(ang) + b * sin(ang);"),
    ("rotary pairs split in halves instead of adjacent channels",
     "int j = c - R + 2 * i;\n            double a = yr[j], b = yr[j + 1];\n"
     "            yr[j] = a * cos(ang) - b * sin(ang);\n            yr[j + 1] = a * sin(ang) + b * cos(ang);",
     "int j = c - R + i;\n            double a = yr[j], b = yr[j + R / 2];\n"
     "            yr[j] = a * cos(ang) - b * sin(ang);\n            yr[j + R / 2] = a * sin(ang) + b * cos(ang);"),
    ("output back-rotation turns forward", "double ang = (inverse ? -p : p) * theta;", "double ang = p * theta;"),
    ("window leaves out the query's own token", "int64_t tau = (int64_t)pos[t] - n_win + 1 + j;",
     "int64_t tau = (int64_t)pos[t] - n_win + j;"),
    ("window ring rows shifted by one", "ring_off + tau % ring_len", "ring_off + (tau + 1) % ring_len"),
    ("e4m3 with four mantissa bits", "int q = e - 4;             /* quantum exponent for 4 significant bits */",
     "int q = e - 5;"),
    ("e4m3 subnormals in steps of 2^-10", "if (q < -9) q = -9;        /* subnormal quantum */",
     "if (q < -10) q = -10;"),
    ("e4m3 ties rounded away from zero",
     "double r = ldexp(round_half_even(ldexp(a, -q)), q);\n    return x < 0 ? -r : r;\n}\n\n/* Row-wise",
     "double r = ldexp(floor(ldexp(a, -q) + 0.5), q);\n    return x < 0 ? -r : r;\n}\n\n/* Row-wise"),
    ("row scale maps the maximum to 240", "amax / 448.0 : 1.0", "amax / 240.0 : 1.0"),
]


def _run_mutant(name, old, new, workdir):
    """Build one mutant and run the pin suite against it; returns (anchor
    found once, pin suite exit code, tail of its output)."""
    src = open(SRC).read()
    if src.count(old) != 1:
        return False, None, ""
    d = os.path.join(workdir, "m%d" % [m[0] for m in MUTATIONS].index(name))
    os.makedirs(d, exist_ok=True)
    mutated = os.path.join(d, "mut.c")
    with open(mutated, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(d, "libmut.so")
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-std=c11", "-shared", "-fPIC", "-o", lib, mutated, "-lm"])
    pins = os.path.join(os.path.dirname(__file__), "test_oracle_pins.py")
    env = dict(os.environ, CSA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", pins],
                       env=env, capture_output=True, text=True, timeout=600)
    return True, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's pin-suite run, several at a time (each is an
    independent process on its own copy of the oracle)."""
    workdir = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(workers) as ex:
        futs = {m[0]: ex.submit(_run_mutant, *m, workdir) for m in MUTATIONS}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(name, old, new, mutant_results):
    found, rc, tail = mutant_results[name]
    assert found, f"mutation anchor not unique/present: {old!r}"
    assert rc != 0, f"no pin failed for mutation '{name}'\n{tail}"
