"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a *copy* of oracle/oracle.c (a dropped term, a wrong sign, an
off-by-one index, a transposed operand), builds it in a temporary directory, and runs the pin
suite (tests/test_oracle_pins.py) against it in a child process: the suite must fail.  A copy
built the same way without a mistake must pass, so the failures come from the mistakes.  The
original file is never written."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "scale dropped": ("s[t - lo] = p->scale * acc;", "s[t - lo] = acc;"),
    "causal limit one too far": ("int pos = T - p->L + i;", "int pos = T - p->L + i + 1;"),
    "causal rows reversed": ("int pos = T - p->L + i;", "int pos = T - 1 - i;"),
    "GTA key from the wrong half of the tied state":
        ("if (j < nope) return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j]);",
         "if (j < nope) return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j + p->d_r]);"),
    "slot within the page off by one":
        ("int slot = t % p->S;\n    size_t tok = (size_t)page * p->S + slot;\n    int grp = h / (p->h_q / p->h_kv);\n    switch",
         "int slot = (t + 1) % p->S;\n    size_t tok = (size_t)page * p->S + slot;\n    int grp = h / (p->h_q / p->h_kv);\n    switch"),
    "query heads interleaved over groups":
        ("int grp = h / (p->h_q / p->h_kv);\n    switch", "int grp = h % p->h_kv;\n    switch"),
    "lse without the running max": ("double lse = m + log(denom);", "double lse = log(denom);"),
    "weights not normalised": ("double w = exp(s[t - lo] - lse);", "double w = exp(s[t - lo] - m);"),
    "combine weight sign": ("double w = exp(part_lse[(size_t)s * rows + r] - L);",
                            "double w = exp(L - part_lse[(size_t)s * rows + r]);"),
    "RoPE rotation sign": ("y[j] = x[j] * c - x[j + half] * s;", "y[j] = x[j] * c + x[j + half] * s;"),
    "GLA rope index shifted": ("return bf16_to_f64(p->c1[tok * p->d_r + (j - p->d)]);",
                               "return bf16_to_f64(p->c1[tok * p->d_r + (j - p->d + 1) % p->d_r]);"),
    "GQA value read from the key cache": ("if (p->variant == ORC_GQA) return bf16_to_f64(p->c1[",
                                          "if (p->variant == ORC_GQA) return bf16_to_f64(p->c0["),
}


def _run_pins(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(src), "-lm"],
                   check=True)
    env = dict(os.environ, KVD_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


def test_unmodified_copy_passes(tmp_path):
    assert _run_pins(tmp_path, "control", open(SRC).read()) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mistake(tmp_path, name):
    orig = open(SRC).read()
    old, new = MUTANTS[name]
    assert orig.count(old) >= 1, f"anchor of '{name}' no longer in oracle.c"
    assert _run_pins(tmp_path, "mutant", orig.replace(old, new, 1)) != 0, f"pins missed: {name}"
