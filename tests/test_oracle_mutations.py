"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a COPY of the oracle's C source (on the CPU), builds it
into a scratch library and runs the pin suite against it: at least one pin must fail.  The
oracle itself is untouched.
"""
import os

import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import osdn_ref

MUTATIONS = {
    # the sign printed in the APF equation (ascent instead of descent)
    "ascent_sign": ("d[i] = rt * d[i] - eta * grad;", "d[i] = rt * d[i] + eta * grad;"),
    # forgetting gate applied to the gradient step as well
    "gate_on_step": ("d[i] = rt * d[i] - eta * grad;", "d[i] = rt * (d[i] - eta * grad);"),
    # beta dropped from the gradient
    "grad_drops_beta": ("-bt * (1.0 - bt * s)", "-(1.0 - bt * s)"),
    # missing normalisation by ||k||^2
    "grad_drops_norm": ("kt[i] * kt[i] / knorm2", "kt[i] * kt[i]"),
    # write key not preconditioned (plain DeltaNet write)
    "write_with_k": ("+= bt * u[j] * kw[i];", "+= bt * u[j] * kt[i];"),
    # k~ built with the key instead of d (.) k
    "ktilde_is_k": ("kw[i] = d[i] * kt[i];", "kw[i] = kt[i];"),
    # readout with the key instead of the query
    "readout_with_k": ("sq += S[(int64_t)j * Dk + i] * qt[i];",
                       "sq += S[(int64_t)j * Dk + i] * kt[i];"),
    # residual without the state term
    "residual_drops_state": ("u[j] = vt[j] - sk;", "u[j] = vt[j];"),
    # <d, k^2> taken as <1, k^2>
    "s_ignores_d": ("s += d[i] * kt[i] * kt[i];", "s += kt[i] * kt[i];"),
    # residual-contraction ratio without its square
    "rho_not_squared": ("rho[th] = (1.0 - bt * s) * (1.0 - bt * s);", "rho[th] = (1.0 - bt * s);"),
}


def _pin_suite(ref):
    yield lambda: pins.test_state_update_is_preconditioned_gradient_step(ref)
    yield lambda: pins.test_preconditioner_step_is_descent_on_surrogate_definition(ref)
    yield lambda: pins.test_brute_force_product(ref, 4, 3, 7)
    yield lambda: pins.test_hand_worked_example(ref, "no_apf")
    yield lambda: pins.test_hand_worked_example(ref, "apf_half")
    yield lambda: pins.test_gated_newton_closed_form(ref, 0.9, 0.7, 0.2, 1.0)
    yield lambda: pins.test_residual_ratio_closed_form(ref)
    yield lambda: pins.test_rho_output_is_the_residual_ratio(ref)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(osdn_ref.SOURCE).read()
    assert old in src, f"mutation anchor for {name} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = osdn_ref.compile_source(str(path), str(tmp_path / f"libmutant_{name}.so"))
    mutant = osdn_ref.Oracle(lib)
    failures = 0
    with np.errstate(all="ignore"):
        for check in _pin_suite(mutant):
            try:
                check()
            except AssertionError:
                failures += 1
    assert failures > 0, f"no pin caught the planted mistake {name!r}"
    os.remove(lib)
