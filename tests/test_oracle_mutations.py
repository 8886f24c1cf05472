"""The oracle's pins catch plausible mistakes (CPU only).

Each case below plants one mistake in a copy of the oracle's C source -- a
dropped gate, a wrong sign, a misplaced factor, a read-out taken at the wrong
time -- builds the copy into its own library and runs the pins of
tests/test_oracle_pins.py against it. Every planted mistake must fail at least
two of them, so that a mistake of that kind in the oracle itself could not pass
the pin suite unnoticed. The committed oracle is never modified.
"""
import importlib.util
import os
import shutil
import sys

import pytest

import test_oracle_pins as pins
from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "gdn2_oracle.c")

# name -> (exact text in the oracle source, replacement)
MUTANTS = {
    # erase reads the decayed state with k instead of b*k (the erase gate dropped)
    "erase_gate_dropped": ("r += p * (b[i] * k[i]);", "r += p * k[i];"),
    # the write gate w does not scale the written value
    "write_gate_dropped": ("double delta = w[j] * v[j] - r;", "double delta = v[j] - r;"),
    # read-out from the decayed state before the write (o_t = P^T q_t instead of S_t^T q_t)
    "readout_before_write": ("oj += s * q[i];", "oj += (s - k[i] * delta) * q[i];"),
    # the rank-one write uses b*k on the key side (factor placement swapped)
    "write_with_erase_factor": ("double s = S[(size_t)i * Dv + j] + k[i] * delta;",
                                "double s = S[(size_t)i * Dv + j] + b[i] * k[i] * delta;"),
    # decay applied as exp(-log_alpha)
    "decay_sign": ("double p = exp(la[i]) * S[(size_t)i * Dv + j];",
                   "double p = exp(-la[i]) * S[(size_t)i * Dv + j];"),
    # adjoint: wrong sign of the read's gradient
    "adjoint_sign_of_dr": ("dr[j] = -acc;", "dr[j] = acc;"),
    # adjoint: the decay is not applied when the state gradient steps back
    "adjoint_decay_missing": ("dS[(size_t)i * Dv + j] = alpha[i] * dp;", "dS[(size_t)i * Dv + j] = dp;"),
}

# the pins, with one parameter set each
PINS = [
    ("bruteforce", lambda o: pins.test_bruteforce_dense_unroll(o, 4, 3, 9)),
    ("golden", pins.test_golden_hand_worked),
    ("kda", pins.test_reduces_to_kda),
    ("gated_deltanet", pins.test_reduces_to_gated_deltanet),
    ("gla_closed_form", pins.test_no_erase_is_gated_linear_attention),
    ("linear_attention", pins.test_no_erase_no_decay_is_linear_attention),
    ("exact_retrieval", pins.test_exact_retrieval),
    ("chunkwise_fwd", lambda o: pins.test_chunkwise_forward_equals_token(o, 16, 37)),
    ("chunkwise_bwd", lambda o: pins.test_chunkwise_backward_equals_token(o, 16, 70)),
    ("finite_differences", pins.test_finite_differences_all_gradients),
    ("decode", pins.test_decode_steps_equal_forward),
]


def _mutant_module(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "the text to mutate must occur once: %r" % old
    pkg = tmp_path / ("oracle_%s" % name)
    pkg.mkdir()
    for f in ("__init__.py", "chunkwise.py"):
        shutil.copy(os.path.join(ROOT, "oracle", f), pkg / f)
    (pkg / "gdn2_oracle.c").write_text(src.replace(old, new))
    modname = "oracle_mutant_%s" % name
    spec = importlib.util.spec_from_file_location(modname, str(pkg / "__init__.py"),
                                                  submodule_search_locations=[str(pkg)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    mod.build()
    return mod


def test_unmutated_copy_passes_every_pin(tmp_path):
    mod = _mutant_module(tmp_path, "none", "int gdn2_oracle_fwd(", "int gdn2_oracle_fwd(")
    for pin_name, pin in PINS:
        pin(mod)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_pins(tmp_path, name):
    mod = _mutant_module(tmp_path, name, *MUTANTS[name])
    failed = []
    for pin_name, pin in PINS:
        try:
            pin(mod)
        except (AssertionError, RuntimeError, FloatingPointError):
            failed.append(pin_name)
    assert len(failed) >= 2, "%s fails only %s" % (name, failed)
    print(name, "fails", failed)
