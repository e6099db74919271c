"""Planted mistakes in copies of the backward-pass oracle: each must fail a pin of
tests/test_oracle_backward.py, and the unmodified copy must pass them all."""

import importlib.util
import inspect
import os

import numpy as np
import pytest

import tests.test_oracle_backward as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "backward.py")

MUTANTS = {
    "state gradient not decayed": ("dM[i] = a * g", "dM[i] = g"),
    "decay gradient without the gate factor": ("dalpha[t] += da * (1.0 - beta[t] * kj)",
                                               "dalpha[t] += da"),
    "write-weight gradient sign": ("dk[t, j] = -da * alpha[t] * beta[t] + db * beta[t]",
                                   "dk[t, j] = da * alpha[t] * beta[t] + db * beta[t]"),
    "softmax backward without its mean": (
        "dsw = k * (dk - np.sum(k * dk, axis=1, keepdims=True))", "dsw = k * dk"),
    "read gradient taken on the state before the token's writes": (
        "        # the read saw the state after token t's writes: M, as it stands now\n"
        "        for j, i in enumerate(idx_r[t]):\n"
        "            dq[t, j] = dy[t] @ M[i]\n",
        "        for j, i in enumerate(idx_r[t]):\n"
        "            dq[t, j] = dy[t] @ np.array([wlog[t, jj] for jj in range(idx_w.shape[1])"
        " if idx_w[t, jj] == i] + [M[i]])[0]\n"),
    "norm backward without the rms term": (
        "dy = r * u - (r ** 3 / d_v) * y * np.sum(u * y, axis=1, keepdims=True)", "dy = r * u"),
    "silu derivative as sigmoid's": ("return g * s, s * (1.0 + g * (1.0 - s))",
                                     "return g * s, s * (1.0 - s)"),
    "second half of the sum skipped": (
        "        np.add.at(dh, (rows, S1 + (idx % S2).ravel()), ds.ravel())\n", ""),
    "undo skipped": ("            M[i] = old  # undo the write\n", ""),
}


def load(text, tmp_path):
    path = tmp_path / "backward_copy.py"
    path.write_text(text)
    spec = importlib.util.spec_from_file_location("backward_copy", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def failing_pins(mod):
    failed = []
    saved = pins.BW
    pins.BW = mod
    old_err = np.seterr(all="ignore")
    try:
        for name, fn in inspect.getmembers(pins, inspect.isfunction):
            if not name.startswith("test_"):
                continue
            params = inspect.signature(fn).parameters
            cases = [{"act": a} for a in ("silu", "sigmoid", "identity")] if "act" in params \
                else [{}]
            for kw in cases:
                try:
                    fn(**kw)
                except AssertionError:
                    failed.append(name)
                    break
    finally:
        pins.BW = saved
        np.seterr(**old_err)
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    assert failing_pins(load(open(SRC).read(), tmp_path)) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_each_mutant_fails_a_pin(tmp_path, mutant):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, mutant
    assert failing_pins(load(src.replace(old, new), tmp_path)), f"no pin catches: {mutant}"
