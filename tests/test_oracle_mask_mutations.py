"""The target-mask oracle's pins catch plausible mistakes: each mutant of
`oracle/target_mask.py` (area weights not normalised, straddling pixels counted whole, the
first partial pixel dropped, a temporal span one frame too long, a temporal sum instead of a
mean, the static mask on the first latent frame only, a wrong shot-length rule, a whole-clip
mask accepted) is loaded from its mutated source on the CPU and must fail at least one pin of
tests/test_oracle_mask_pins.py."""
import importlib.util
import inspect

import pytest

import oracle
from oracle import target_mask
import test_oracle_mask_pins as pins
from conftest import read_golden

SRC = target_mask.__file__

MUTANTS = {
    "weights not normalised": ("W[o, i] = ov / step", "W[o, i] = ov"),
    "straddling pixels counted whole": ("ov = min(hi, i + 1) - max(lo, i)", "ov = 1.0"),
    "first partial pixel dropped": ("range(int(np.floor(lo)),", "range(int(np.ceil(lo)),"),
    "span one frame too long": ("t0, t1 = f * tau, min((f + 1) * tau, L)",
                                "t0, t1 = f * tau, min((f + 1) * tau + 1, L)"),
    "temporal sum": ("out[f] = down[t0:t1].mean(axis=0)", "out[f] = down[t0:t1].sum(axis=0)"),
    "static mask on one latent frame": (
        "return np.repeat(down, F_lat, axis=0)",
        "return np.concatenate([down, np.zeros((F_lat - 1,) + down.shape[1:])])"),
    "shot length 17n+4": ("(L - 5) % 17 == 0", "(L - 4) % 17 == 0"),
    "whole-clip mask accepted": ("(F_in == 1 or F_in == L)", "(F_in == 1 or F_in >= L)"),
}

EXPORTED = ("area_weights", "mask_length_ok", "prepare_target_mask", "shot_length_ok")


def _load_mutant(src: str):
    spec = importlib.util.spec_from_loader("oracle.target_mask_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src, SRC + " (mutant)", "exec"), mod.__dict__)
    return mod


def _run_pins():
    """Names of the pins that fail."""
    fixtures = {"golden_rule": read_golden("tara_rule_pages.txt")}
    failed = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        args = [fixtures[a] for a in inspect.signature(fn).parameters]
        try:
            fn(*args)
        except (AssertionError, ValueError, IndexError, pytest.fail.Exception):
            failed.append(name)
    return failed


def _install(monkeypatch, mod):
    for name in EXPORTED:
        monkeypatch.setattr(oracle, name, getattr(mod, name))


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(mutant, monkeypatch):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: %s" % mutant
    _install(monkeypatch, _load_mutant(src.replace(old, new)))
    assert _run_pins(), "mutant '%s' passed every pin" % mutant


def test_unmutated_source_passes_every_pin(monkeypatch):
    _install(monkeypatch, _load_mutant(open(SRC).read()))
    assert _run_pins() == []
