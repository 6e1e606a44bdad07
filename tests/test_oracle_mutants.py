"""The oracle's pins catch plausible mistakes: each mutant below is a copy of
nm_oracle.c with one deliberate error, compiled on the CPU and loaded by the
oracle's pin tests in a subprocess, which must fail.  The unmodified source
built the same way must pass (the harness itself works)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nm_oracle.c")
PINS = [os.path.join(ROOT, "tests", "test_oracle.py"), os.path.join(ROOT, "tests", "test_oracle_tile.py")]

MUTANTS = {
    "compress tie rule reversed": ("(aq == ap && q < p)", "(aq == ap && q > p)"),
    "compress keeps on >= instead of >": ("if (aq > ap ||", "if (aq >= ap ||"),
    "compress keeps N+1": ("if (ahead < N) {", "if (ahead <= N) {"),
    "tile score is the max, not the sum":
        ("score[p] += magnitude(W, dtype, r * k + g * M + p);",
         "score[p] = fmax(score[p], magnitude(W, dtype, r * k + g * M + p));"),
    "tile tie rule reversed": ("(score[q] == score[p] && q < p)", "(score[q] == score[p] && q > p)"),
    "tile ignores its last row": ("for (int64_t r = r0; r < r1; ++r) score[p]", "for (int64_t r = r0; r < r1 - 1; ++r) score[p]"),
    "gemm drops the last k": ("for (int64_t kk = 0; kk < K; ++kk)\n                acc += (int64_t)X",
                              "for (int64_t kk = 0; kk + 1 < K; ++kk)\n                acc += (int64_t)X"),
    "gemm reads the weight transposed": ("(int64_t)Wm[n * K + kk]", "(int64_t)Wm[kk * n_out + n]"),
    "scale taken from the wrong channel": ("float s = scale[n];", "float s = scale[n_out - 1 - n];"),
    "fp16 decoder exponent off by one": ("ldexp((double)(m | 0x400), e - 25)", "ldexp((double)(m | 0x400), e - 24)"),
    "bias added before the scale": ("if (scale) v = v * scale[n];\n            if (bias) v = v + bias[n];",
                                    "if (bias) v = v + bias[n];\n            if (scale) v = v * scale[n];"),
    "int8 rounding truncates": ("q[i] = sat_s8((double)rintf(p));", "q[i] = sat_s8((double)truncf(p));"),
    "int8 path: GELU before the bias":
        ("const double g = gelu_erf((double)v);",
         "const double g = gelu_erf((double)v - (bias ? bias[n] : 0.0f)) + (bias ? bias[n] : 0.0f);"),
    "float path: GELU before the bias":
        ("if (bias) v += (double)bias[n];\n            pre[i] = act == 1 ? gelu_erf(v) : v;",
         "pre[i] = act == 1 ? gelu_erf(v) : v;\n            if (bias) pre[i] += (double)bias[n];"),
    "float path: bias before the scale":
        ("if (scale) v *= (double)scale[n];\n            if (bias) v += (double)bias[n];",
         "if (bias) v += (double)bias[n];\n            if (scale) v *= (double)scale[n];"),
    "GELU drops the 1/2":("static double gelu_erf(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }",
                           "static double gelu_erf(double x) { return x * (1.0 + erf(x / sqrt(2.0))); }"),
}


def _build(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                           "-o", str(lib), str(src), "-lm"])
    return str(lib)


def _run_pins(lib):
    env = dict(os.environ, NM_ORACLE_LIB=lib, OMP_NUM_THREADS="4")
    return subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_unmodified_oracle_passes_through_the_harness(tmp_path):
    r = _run_pins(_build(tmp_path, "original", open(SRC).read()))
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site not found exactly once: {old!r}"
    r = _run_pins(_build(tmp_path, "mutant", text.replace(old, new)))
    assert r.returncode != 0, f"no pin failed for the mutant '{name}'"
