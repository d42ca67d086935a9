"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong sign, a wrong index or bound, a transposed operand), builds it,
points the ``oracle`` package at it, and runs the pins of ``test_oracle.py``:
at least one pin must fail.  The shipped oracle is restored afterwards.
"""
import os

import numpy as np
import pytest

import oracle
import test_oracle as pins

# (name, text in ratp_oracle.c, replacement); only the first occurrence is
# changed, which is the function named in the case
MUTATIONS = [
    ("scan drops (1-g)", "state = g[i] * state + (1.0 - g[i]) * x[i];", "state = g[i] * state + x[i];"),
    ("scan sign of g", "state = g[i] * state + (1.0 - g[i]) * x[i];", "state = g[i] * state + (1.0 + g[i]) * x[i];"),
    ("scan initial state", "double state = 0.0;                      /* h_{-1} = 0 */",
     "double state = 1.0;"),
    ("dilated positions off by one", "for (long j = D - 1; j < t; j += D)", "for (long j = D; j < t; j += D)"),
    ("window one position short", "        long lo = t - W + 1;\n        if (lo < 0) lo = 0;",
     "        long lo = t - W + 2;\n        if (lo < 0) lo = 0;"),
    ("softmax scale dropped", "const double scale = 1.0 / sqrt((double)Dh);", "const double scale = 1.0;"),
    ("scores against values", "const double* kj = hk + (keys[i] * H + h) * Dh;",
     "const double* kj = hv + (keys[i] * H + h) * Dh;"),
    ("decode appends at the wrong position", "            if (t % Dd == Dd - 1) {\n                long s = t / Dd;",
     "            if (t % Dd == 0) {\n                long s = t / Dd;"),
    ("chunk-local restart position", "if (L > 0 && t % L == 0) state = 0.0;", "if (L > 0 && t % L == 1) state = 0.0;"),
    ("decode restart position", "if (L > 0 && t % L == 0) {", "if (L > 0 && t % L == 1) {"),
    ("look-back window one too long", "long j0 = t - L + 1;", "long j0 = t - L;"),
]

PINS = [
    pins.test_scan_hand_fixture,
    pins.test_scan_gate_zero_is_identity,
    lambda: pins.test_scan_constant_gate_geometric_sum(0.9),
    pins.test_scan_constant_gate_unit_input,
    pins.test_scan_associative_composition,
    pins.test_scan_reset_every_token_is_input_weighting,
    lambda: pins.test_scan_reset_constant_gate_unit_input(16),
    lambda: pins.test_scan_reset_blocks_are_independent(7),
    pins.test_scan_window_one_token_is_input_weighting,
    lambda: pins.test_scan_window_covering_sequence_is_full(19),
    lambda: pins.test_scan_window_constant_gate_closed_form(16, 0.95),
    lambda: pins.test_scan_window_matches_blocks_and_suffix_form(4),
    pins.test_key_set_hand_fixture,
    pins.test_key_set_matches_predicate,
    pins.test_key_set_count_closed_form,
    pins.test_attention_hand_fixture,
    pins.test_attention_dense_equals_sdpa,
    lambda: pins.test_attention_window_covering_sequence_is_dense(5),
    pins.test_attention_dilation_beyond_sequence_is_self,
    lambda: pins.test_attention_enumeration_equals_mask(16, 4, 3),
    pins.test_cache_layout_hand_fixture,
    lambda: pins.test_decode_continues_prefill(4, 2, None),
    lambda: pins.test_decode_chunk_local_continues_prefill(5, 13),
]


@pytest.fixture
def mutated_oracle(tmp_path):
    saved = (oracle._SRC, oracle._LIB, oracle._lib)
    src = open(oracle._SRC).read()

    def load(old, new):
        assert src.count(old) >= 1, old
        path = tmp_path / ("m%d.c" % len(os.listdir(tmp_path)))
        path.write_text(src.replace(old, new, 1))
        oracle._SRC, oracle._LIB, oracle._lib = str(path), str(path) + ".so", None
        oracle._load()

    yield load
    oracle._SRC, oracle._LIB, oracle._lib = saved


def _failing_pins():
    failed = []
    for i, pin in enumerate(PINS):
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError, IndexError):
            failed.append(i)
    return failed


def test_shipped_oracle_passes_every_pin():
    assert _failing_pins() == []


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(mutated_oracle, name, old, new):
    mutated_oracle(old, new)
    np.seterr(all="ignore")
    assert _failing_pins(), "no pin caught: %s" % name
