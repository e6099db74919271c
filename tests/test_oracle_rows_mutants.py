"""Planted mistakes in copies of the checkpoint-row oracle: each must fail at least one pin of
tests/test_oracle_rows.py, and the unmodified copy must pass them all."""

import importlib.util
import inspect
import os

import numpy as np
import pytest

import tests.test_oracle_rows as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rows.py")

MUTANTS = {
    "ties to the odd code": ("code = i if i % 2 == 0 else i + 1",
                             "code = i + 1 if i % 2 == 0 else i"),
    "no saturation": ("    if a >= E4M3_MAX:\n        code = 126",
                      "    if a >= 1e300:\n        code = 126"),
    "E4M3 scale over 480": ("E4M3_MAX = 448.0", "E4M3_MAX = 480.0"),
    "signed zero kept": ("0x80 if neg and code != 0 else 0", "0x80 if neg else 0"),
    "subnormal exponent off by one": ("return sign * 2.0 ** -6 * (m / 8.0)",
                                      "return sign * 2.0 ** -7 * (m / 8.0)"),
    "bf16 truncates": ("((u + 0x7FFF + keep_odd) >> 16)", "((u) >> 16)"),
    "bf16 ties away from zero": ("((u + 0x7FFF + keep_odd) >> 16)", "((u + 0x8000) >> 16)"),
    "int4 nibbles swapped": ("codes[r] = nib[0::2] | (nib[1::2] << 4)",
                             "codes[r] = nib[1::2] | (nib[0::2] << 4)"),
    "int4 rounds half away from zero": ("np.clip(np.rint(q)",
                                        "np.clip(np.trunc(q + np.copysign(0.5, q))"),
    "int4 sign extension wrong": ("np.where(k >= 8, k - 16, k)", "np.where(k >= 8, k - 15, k)"),
    "int4 scale over 8": ("INT4_MAX = 7\n", "INT4_MAX = 8\n"),
    "tiny scales kept": ("return s if s >= FLT_MIN else np.float32(0)", "return s"),
}


def load(src_text, tmp_path, name):
    path = tmp_path / f"{name}.py"
    path.write_text(src_text)
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def failing_pins(mod):
    failed = []
    saved = pins.R
    pins.R = mod
    old_err = np.seterr(all="ignore")  # a mutant may overflow; the pins judge the result
    try:
        for name, fn in inspect.getmembers(pins, inspect.isfunction):
            if not name.startswith("test_"):
                continue
            params = inspect.signature(fn).parameters
            cases = [{"fmt": f} for f in ("e4m3", "int4")] if "fmt" in params else [{}]
            for kw in cases:
                try:
                    fn(**kw)
                except Exception:  # noqa: BLE001 - any failure of a pin counts
                    failed.append(name)
                    break
    finally:
        pins.R = saved
        np.seterr(**old_err)
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    assert failing_pins(load(open(SRC).read(), tmp_path, "rows_copy")) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_each_mutant_fails_a_pin(tmp_path, mutant):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, mutant
    mod = load(src.replace(old, new), tmp_path, "rows_mutant")
    assert failing_pins(mod), f"no pin catches: {mutant}"
