"""Sensitivity of the oracle's pins.

Each mutant below plants one plausible mistake in a copy of the oracle's C source: a
flipped order, a transposed or lagged index, a dropped or complemented term, a wrong
normalisation or activation.  The pin suite (test_oracle_pins.py) runs against each
mutant's build in a child process and must fail on every one of them, while it passes on
an unmodified copy built the same way.  The mistakes are planted in the oracle, on the
CPU; the product's kernels are not involved.

The statements the mutants violate: "Sparse Delta Memory: Scaling the State of Linear RNNs
through Sparsity" (paper.rainbus.top summary), method steps 1-4; the SDM write-up on
ai-paper-analysis.pages.dev, sections 步骤 1-4.
"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# name -> (text of the oracle source, its replacement)
MUTANTS = {
    # step 1: the order (score descending, index ascending) and the slot numbering
    "scores_ascending": ("if (a->s != b->s) return a->s > b->s;",
                         "if (a->s != b->s) return a->s < b->s;"),
    "ties_to_highest_index": ("return a->i < b->i;", "return a->i > b->i;"),
    "plus_zero_before_minus_zero": (
        "if (a->s != b->s) return a->s > b->s;",
        "if (a->s != b->s) return a->s > b->s;\n"
        "    if (signbit(a->s) != signbit(b->s)) return !signbit(a->s);"),
    "flat_index_transposed": ("c.i = h1[a].i * (int64_t)S2 + h2[b].i;",
                              "c.i = h2[b].i * (int64_t)S1 + h1[a].i;"),
    "one_candidate_short_per_half": ("const int K1 = K < S1 ? K : S1;",
                                     "const int K1 = K < S1 ? (K > 1 ? K - 1 : K) : S1;"),
    # step 1: the slot weights
    "weights_not_normalised": ("for (int j = 0; j < K; ++j) wt[j] /= total;", ""),
    "weights_at_half_temperature": ("wt[j] = exp((double)sel[j].s - s0);",
                                    "wt[j] = exp(0.5 * ((double)sel[j].s - s0));"),
    # step 2: the gated delta write
    "decay_dropped": ("const double m_tilde = a_t * m[c];", "const double m_tilde = m[c];"),
    "delta_against_undecayed_row": ("((double)v_t[c] - m_tilde)", "((double)v_t[c] - m[c])"),
    "write_weight_dropped": ("m[c] = m_tilde + b_t * k_i * (", "m[c] = m_tilde + b_t * ("),
    "beta_complemented": ("m[c] = m_tilde + b_t * k_i * (",
                          "m[c] = m_tilde + (1.0 - b_t) * k_i * ("),
    # step 2, coupled reading: the shared prediction
    "coupled_prediction_undecayed": ("pred[c] += kj * (a_t * row[c]);", "pred[c] += kj * row[c];"),
    "coupled_prediction_unweighted": ("pred[c] += kj * (a_t * row[c]);",
                                      "pred[c] += a_t * row[c];"),
    # the undo log of the in-place update: the row as the write found it
    "undo_log_of_decayed_row": ("wlog[((long)t * W + j) * d_v + c] = m[c];",
                                "wlog[((long)t * W + j) * d_v + c] = a_t * m[c];"),
    # step 3: the sparse read
    "read_weight_dropped": ("acc[c] += q_i * m[c];", "acc[c] += m[c];"),
    "read_uses_previous_tokens_slots": ("const int32_t i = idx_r[(long)t * R + j];",
                                       "const int32_t i = idx_r[(long)(t > 0 ? t - 1 : 0) * R + j];"),
    # step 4: RMSNorm and the output gate
    "norm_by_sum_not_mean": ("sqrt(ss / (double)d_v + eps)", "sqrt(ss + eps)"),
    "silu_as_sigmoid": ("if (act == 0) gate = x / (1.0 + exp(-x));",
                        "if (act == 0) gate = 1.0 / (1.0 + exp(-x));"),
    "gamma_ignored": ("const double w = gamma ? (double)gamma[c] : 1.0;",
                      "const double w = 1.0;"),
}

# Runs the pin suite with the oracle built from another source file.
RUNNER = r"""
import sys
sys.path.insert(0, sys.argv[4])
import oracle
oracle._SRC, oracle._LIB_PATH, oracle._lib = sys.argv[1], sys.argv[2], None
import pytest
sys.exit(pytest.main([sys.argv[3], "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"]))
"""


def run_pins(src_path: str, lib_path: str) -> subprocess.CompletedProcess:
    return subprocess.run([sys.executable, "-c", RUNNER, src_path, lib_path, PINS, ROOT],
                          cwd=ROOT, capture_output=True, text=True, timeout=600)


def test_every_mutant_fails_a_pin_and_the_unmodified_copy_passes(tmp_path):
    source = open(oracle._SRC).read()
    jobs = {"unmodified": source}
    for name, (old, new) in MUTANTS.items():
        assert source.count(old) == 1, f"{name}: the text to mutate is not unique"
        jobs[name] = source.replace(old, new)
    paths = {}
    for name, text in jobs.items():
        src = tmp_path / f"{name}.c"
        src.write_text(text)
        paths[name] = (str(src), str(tmp_path / f"lib{name}.so"))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        results = dict(zip(paths, pool.map(lambda p: run_pins(*p), paths.values())))

    control = results.pop("unmodified")
    assert control.returncode == 0, control.stdout[-2000:] + control.stderr[-2000:]
    survivors = [n for n, r in results.items() if r.returncode == 0]
    assert not survivors, f"mutants no pin detects: {survivors}"
    # a detection is a failed pin (exit code 1), not a build error or a crash
    other = {n: r.returncode for n, r in results.items() if r.returncode != 1}
    assert not other, f"mutants that did not run to a failed pin: {other}"


# Mistakes planted in the Python undo (a replay of the log): each must fail an undo pin.
UNDO_MUTANTS = {
    "replayed_forwards": ("for t in range(T - 1, -1, -1):", "for t in range(T):"),
    "last_token_skipped": ("for t in range(T - 1, -1, -1):", "for t in range(T - 2, -1, -1):"),
    "first_token_skipped": ("for t in range(T - 1, -1, -1):", "for t in range(T - 1, 0, -1):"),
}


@pytest.mark.parametrize("mutant", sorted(UNDO_MUTANTS))
def test_every_undo_mutant_fails_a_pin(mutant, monkeypatch):
    import inspect
    import textwrap

    import numpy as np

    import tests.test_oracle_pins as pins
    old, new = UNDO_MUTANTS[mutant]
    src = textwrap.dedent(inspect.getsource(oracle.undo))
    assert src.count(old) == 1
    ns = {"np": np}
    exec(src.replace(old, new), ns)  # noqa: S102 - a planted copy of the oracle's own code
    monkeypatch.setattr(oracle, "undo", ns["undo"])
    caught = 0
    for pin in (pins.test_undo_restores_the_starting_state,
                pins.test_undo_of_three_decays_of_one_slot):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no undo pin detects {mutant}"
