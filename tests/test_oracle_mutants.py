"""The pins must catch plausible mistakes: each mutant oracle (one planted error,
compiled with -DORACLE_MUTANT=k) has to fail at least one pin."""
import pytest

import oracle
import tests.test_oracle_pins as pins
from selective_diagonal_state_b200 import synthetic as S

MUTANTS = {
    1: "two-endpoint (beta) term dropped",
    2: "rotation direction flipped",
    3: "readout C taken from the wrong group",
    4: "rank index of B transposed",
    5: "sign of dtheta flipped",
    6: "dbeta uses W_t instead of W_{t-1}",
    7: "lam * dgamma missing from ddt",
    8: "adjoint uses A instead of A^T",
    9: "feedthrough D u dropped",
    10: "static rows decay by e^{dt a} instead of e^{a}",
    11: "static rows' decay gradient weighted by dt",
    12: "sign of the per-token angle gradient flipped",
    13: "ZOH write's dt-derivative taken as phi1 instead of e^mu",
    14: "ZOH backward applies Z instead of Z^T to a pair's adjoint",
}

PIN_CALLS = [
    lambda: pins.test_recurrence_equals_quadratic_masked_form(dict()),
    lambda: pins.test_recurrence_equals_quadratic_masked_form(dict(rank_in=3, rank_out=2, n_pairs=1)),
    lambda: pins.test_recurrence_equals_quadratic_masked_form(dict(rank_in=2, rank_out=2, ngroups=1)),
    lambda: pins.test_recurrence_equals_quadratic_masked_form(dict(nheads=4, ngroups=2, batch=1)),
    lambda: pins.test_real_2x2_blocks_equal_complex_diagonal(dict()),
    lambda: pins.test_lti_equals_vandermonde_convolution(),
    lambda: pins.test_single_step_closed_form(),
    lambda: pins.test_gradients_match_central_differences(dict(rank_in=2, rank_out=2, ngroups=1)),
    lambda: pins.test_gradients_match_central_differences(dict(rank_in=2, rank_out=2, ngroups=2)),
    lambda: pins.test_gradients_match_central_differences(dict(nheads=4, ngroups=2, headdim=1,
                                                               seqlen=8)),
    lambda: pins.test_static_rows_lti_vandermonde(),
    lambda: pins.test_static_row_gradients_match_central_differences(S.DECAY_PER_COORD),
    lambda: pins.test_per_token_angles_equal_complex_modes(),
    lambda: pins.test_per_token_angle_gradients_match_central_differences(),
    lambda: pins.test_zoh_equals_matrix_exponential(dict()),
    lambda: pins.test_zoh_gradients_match_central_differences(dict()),
]


@pytest.mark.parametrize("k", sorted(MUTANTS))
def test_mutant_is_caught(k, monkeypatch):
    path = oracle.build(extra_flags=(f"-DORACLE_MUTANT={k}",))
    lib = oracle._load(path)
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = 0
    for call in PIN_CALLS:
        try:
            call()
        except AssertionError:
            caught += 1
    assert caught > 0, f"mutant {k} ({MUTANTS[k]}) passed every pin"
