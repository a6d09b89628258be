"""Planted mistakes in the oracle must be caught by its pins.

Each mutation is a plausible conceptual error (a dropped term, a wrong sign or
index, exchanged operands) applied consistently to every oracle route, so
route-against-route agreement alone cannot catch it; the external pins
(closed forms, limits, exact arithmetic, grouping, chunk invariance) must.
Everything runs on the CPU; the mutation switch is reset after each test.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import ssd_oracle as O
from tests import test_oracle_pins as pins

MUTATIONS = {
    1: "drop D",
    2: "decay includes a_s",
    3: "B and C exchanged",
    4: "head->group as h % G",
    5: "exp(-a)",
    6: "inter-chunk term without exp(cum_t)",
    7: "chunk state without decay weights",
    8: "per-state decay read from n+1",
    9: "output before the state update",
}

PIN_FUNCS = [
    ("lti", lambda: [pins.test_lti_closed_form_convolution(False),
                     pins.test_lti_closed_form_convolution(True)]),
    ("linear_attention", lambda: [pins.test_zero_decay_is_causal_linear_attention(G, H)
                                  for G, H in [(1, 3), (2, 4)]]),
    ("memoryless", pins.test_memoryless_limit),
    ("exact", pins.test_exact_rational_brute_force),
    ("golden", pins.test_golden_impulse_response_decay_085),
    ("grouping", lambda: [pins.test_grouped_bc_equals_replicated(False),
                          pins.test_grouped_bc_equals_replicated(True)]),
    ("chunk_invariance", lambda: [pins.test_chunked_is_chunk_invariant(ps, 24, [1, 3, 6, 8, 12, 24])
                                  for ps in (False, True)]),
]


@pytest.fixture
def clean_mutation():
    O.set_mutation(0)
    yield
    O.set_mutation(0)


def _failing_pins():
    failed = []
    for name, fn in PIN_FUNCS:
        try:
            with np.errstate(all="ignore"):
                fn()
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(name)
    return failed


def test_pins_pass_without_mutation(clean_mutation):
    assert _failing_pins() == []


@pytest.mark.parametrize("m", sorted(MUTATIONS))
def test_planted_mistake_is_caught(clean_mutation, m):
    O.set_mutation(m)
    failed = _failing_pins()
    O.set_mutation(0)
    assert failed, f"mutation {m} ({MUTATIONS[m]}) passed every pin"


BACKWARD_MUTATIONS = {
    1: "loss on the final state dropped",
    2: "adjoint picks up B instead of C",
    3: "dx without the D term",
    4: "dB from the state instead of the adjoint",
    5: "dC from the state before the step",
    6: "da without the decay factor",
    7: "adjoint not decayed between steps",
}


@pytest.mark.parametrize("m", sorted(BACKWARD_MUTATIONS), ids=lambda m: BACKWARD_MUTATIONS[m])
def test_backward_pins_catch_planted_mistake(m):
    """Each planted mistake in the oracle's backward makes its finite-difference
    pin fail (the pin differentiates the forward oracle, which the planted
    mistake does not touch)."""
    from tests import test_oracle_backward as bpins
    O.set_backward_mutation(m)
    try:
        caught = False
        for per_state in (False, True):
            try:
                bpins.test_backward_matches_finite_differences(per_state, 1, 2)
            except AssertionError:
                caught = True
        assert caught, BACKWARD_MUTATIONS[m]
    finally:
        O.set_backward_mutation(0)
