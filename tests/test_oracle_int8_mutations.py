"""The INT8-QK^T oracle's pins catch plausible mistakes: each mutant of `oracle/int8_qk.py`
(ties rounded away from zero, a wrong code range or scale, a wrong K block size, V quantised
too, Q and K swapped, blocks' scales misassigned) is loaded from its mutated source on the CPU
and must fail at least one pin of tests/test_oracle_int8_pins.py."""
import importlib.util
import inspect
import os

import pytest

from oracle import int8_qk
import test_oracle_int8_pins as pins

SRC = int8_qk.__file__

MUTANTS = {
    "ties away from zero": ("codes = np.rint(prod)", "codes = np.floor(prod + np.float32(0.5))"),
    "codes up to 128": ("QMAX = np.float32(127.0)", "QMAX = np.float32(128.0)"),
    "scale off by one": ("(amax / QMAX).astype(np.float32)",
                         "(amax / np.float32(126.0)).astype(np.float32)"),
    "K blocks of 64": ("KBLOCK = 128", "KBLOCK = 64"),
    "V quantised too": ("vd = _widen_f32(v_raw, dtype).astype(np.float64)",
                        "vd = dequantise_q(*quantise_q(_widen_f32(v_raw, dtype)))"),
    "Q and K swapped": ("return attention_rows(qd, kd, vd,", "return attention_rows(kd, qd, vd,"),
    "block scales reversed": ("np.repeat(scales.astype(np.float64), KBLOCK, axis=2)",
                              "np.repeat(scales.astype(np.float64)[:, :, ::-1], KBLOCK, axis=2)"),
    "floor ignored": ("live = amax > AMAX_FLOOR", "live = amax > 0"),
}


def _load_mutant(src: str):
    spec = importlib.util.spec_from_loader("oracle.int8_qk_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src, SRC + " (mutant)", "exec"), mod.__dict__)
    return mod


def _pins():
    return [fn for name, fn in inspect.getmembers(pins, inspect.isfunction)
            if name.startswith("test_")]


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(mutant, monkeypatch):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: %s" % mutant
    monkeypatch.setattr(pins, "Q8", _load_mutant(src.replace(old, new)))
    failed = []
    for fn in _pins():
        try:
            fn()
        except (AssertionError, ValueError, RuntimeError, IndexError):
            failed.append(fn.__name__)
    assert failed, "mutant '%s' passed every pin" % mutant


def test_unmutated_source_passes_every_pin(monkeypatch):
    monkeypatch.setattr(pins, "Q8", _load_mutant(open(SRC).read()))
    for fn in _pins():
        fn()
