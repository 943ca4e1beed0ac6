"""Planted mistakes in the backward oracle (a copy of oracle/backward.py with one edit each)
must each fail a backward pin: finite differences of the forward C oracle, or torch
autograd through the printed operator. CPU only."""
import os
import types

import pytest

import oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "backward.py")

MUTANTS = {
    "dv sign of branch 2": ("dv = a1.T @ dO - lam * (a2.T @ dO)", "dv = a1.T @ dO + lam * (a2.T @ dO)"),
    "softmax backward without the row sum": (
        "ds1 = a1 * (da1 - (a1 * da1).sum(axis=-1, keepdims=True))", "ds1 = a1 * da1"),
    "dK not transposed": ("dk1, dk2 = ds1.T @ q1 * sc, ds2.T @ q2 * sc", "dk1, dk2 = ds2.T @ q1 * sc, ds2.T @ q2 * sc"),
    "dlambda sign": ("dlam = -float(np.sum(dO * (a2 @ v)))", "dlam = float(np.sum(dO * (a2 @ v)))"),
    "dlambda from branch 1": ("dlam = -float(np.sum(dO * (a2 @ v)))", "dlam = -float(np.sum(dO * (a1 @ v)))"),
    "norm backward without the projection": (
        "return scale / r * (dy - o * dot / (n * r * r))", "return scale / r * dy"),
    "norm mean over the wrong count": (
        "return scale / r * (dy - o * dot / (n * r * r))", "return scale / r * (dy - o * dot / (r * r))"),
    "scale 1/d": ("sc = 1.0 / np.sqrt(d)\n    a1", "sc = 1.0 / d\n    a1"),
    "GQA KV head of the wrong pair": ("g = (2 * p) // group", "g = p % k.shape[2]"),
    "causal mask off by one": ("m &= j <= pos", "m &= j < pos + 2"),
    "window bound": ("m &= j > pos - window", "m &= j >= pos - window"),
    "lambda vector e2 sign": ("-dlam * e2 * lk2, -dlam * e2 * lq2", "dlam * e2 * lk2, -dlam * e2 * lq2"),
    "lambda vector swapped": ("dlam * e1 * lk1, dlam * e1 * lq1", "dlam * e1 * lq1, dlam * e1 * lk1"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    monkeypatch.setattr(P, "OB", _mutant(*MUTANTS[name]))
    failed = 0
    for pin in (P.pin_backward_finite_differences, P.pin_backward_autograd):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed, f"no backward pin caught: {name}"
