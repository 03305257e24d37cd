"""The oracle's pins catch plausible mistakes: each mutant of the oracle's C source (a flipped
sign, a dropped term, swapped query/key roles, a wrong index, a transposed operand) is
compiled on the CPU and must fail at least one pin of tests/test_oracle_pins.py.
Nothing here touches a GPU."""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins
from conftest import read_golden

SRC = os.path.join(os.path.dirname(oracle.__file__), "tara_oracle.c")

MUTANTS = {
    "penalty sign": ("return -oracle_penalty(dt, window, falloff, strength, cap);",
                     "return oracle_penalty(dt, window, falloff, strength, cap);"),
    "scale dropped": ("double sj = dot * scale + oracle_bias(",
                      "double sj = dot + oracle_bias("),
    "query/key roles swapped": ("if (seg[i] != ROLE_TARGET) return 0.0;",
                                "if (seg[j] != ROLE_TARGET) return 0.0;"),
    "window dropped": ("double x = dt - window;", "double x = dt;"),
    "falloff multiplies": ("x = x / falloff;", "x = x * falloff;"),
    "cap ignored": ("return p < cap ? p : cap;", "return p;"),
    "mask weight dropped": ("double b = (double)m[i] * log(gain9[p - 1]);",
                            "double b = log(gain9[p - 1]);"),
    "picture index off by one": ("double b = (double)m[i] * log(gain9[p - 1]);",
                                 "double b = (double)m[i] * log(gain9[p % 9]);"),
    "extra binding reuses the first gains": ("* log(extra->gains[9 * k + p - 1]);",
                                             "* log(gain9[p - 1]);"),
    "extra binding ignores its mask": ("b += (double)extra->m[k * extra->m_len + mo + i] *",
                                       "b += 1.0 *"),
    "extra bindings replace instead of add": ("b += (double)extra->m[", "b = (double)extra->m["),
    "values used as keys": ("dot += q[k] * widen(K, dtype, head + j * D + k);",
                            "dot += q[k] * widen(V, dtype, head + j * D + k);"),
    "lse without max": ("LSE_out[r] = M + log(l);", "LSE_out[r] = log(l);"),
    "signed time difference": ("double dt = fabs((double)time_s[i] - (double)time_s[j]);",
                               "double dt = (double)time_s[i] - (double)time_s[j];"),
    "guide/picture roles swapped": ("if (seg[j] == ROLE_GUIDE) {", "if (seg[j] == ROLE_PICTURE) {"),
    # each rule parameter replaced by its printed default
    "falloff hard-coded to its default": ("x = x / falloff;", "x = x / 0.25;"),
    "window hard-coded to its default": ("double x = dt - window;", "double x = dt - 0.20;"),
    "strength hard-coded to its default": ("double p = strength * x * x;", "double p = 2.0 * x * x;"),
    "cap hard-coded to its default": ("return p < cap ? p : cap;", "return p < 6.0 ? p : 6.0;"),
}


def _pin_calls(golden):
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or "packer" in name:
            continue
        params = inspect.signature(fn).parameters
        if "which" in params:
            calls += [(name + "[%s]" % w, lambda fn=fn, w=w: fn(w)) for w in ("strength0", "cap0")]
        elif "golden_rule" in params:
            calls.append((name, lambda fn=fn: fn(golden)))
        else:
            calls.append((name, fn))
    return calls


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: %s" % mutant
    path_c = tmp_path / "mutant.c"
    path_so = tmp_path / "libmutant.so"
    path_c.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", "-o",
                           str(path_so), str(path_c), "-lm"])
    golden = read_golden("tara_rule_pages.txt")
    saved = oracle._load()
    oracle._lib = oracle._bind(ctypes.CDLL(str(path_so)))
    failed = []
    try:
        for name, call in _pin_calls(golden):
            try:
                call()
            except (AssertionError, ValueError, RuntimeError):
                failed.append(name)
    finally:
        oracle._lib = saved
    assert failed, "mutant '%s' passed every pin" % mutant


def test_unmutated_source_passes_every_pin():
    golden = read_golden("tara_rule_pages.txt")
    for name, call in _pin_calls(golden):
        call()
