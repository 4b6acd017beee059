"""The fp64 oracle against closed forms, brute force, library routines,
invariants and hand-worked examples (CPU only)."""

import numpy as np
import pytest

import oracle_pins as pins
from selective_state_space_causal_b200 import synth


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_decode_invariant_long(orc):
    pins.check_decode_invariant(orc, k_steps=(1000,))


def test_closed_form_long_sequence(orc):
    pins.check_closed_form(orc, L=8192, D=3, N=16)


def test_thread_count_does_not_change_results(orc):
    p, a = pins._rand_layer(61, 300, 16, 16, 4)
    cu = np.array([0, 100, 130, 300], dtype=np.int64)
    n0 = orc.num_threads()
    try:
        orc.set_num_threads(1)
        y1 = pins._layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p, cu)
        orc.set_num_threads(max(2, n0))
        y2 = pins._layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p, cu)
    finally:
        orc.set_num_threads(n0)
    for u, v in zip(y1, y2):
        assert np.array_equal(u, v)


def test_synthetic_delta_range():
    """softplus(dt + dt_bias) of the input recipe stays in [1e-3, 1e-1]."""
    prm = synth.make_params(0, 512)
    act = synth.make_activations(0, 256, 512, bf16=True)
    delta = np.logaddexp(0.0, act["dt"].astype(np.float64) + prm.dt_bias[None, :])
    assert delta.min() >= 1e-3 and delta.max() <= 1e-1, (delta.min(), delta.max())


def test_packed_lengths_recipe():
    lens = synth.sample_lengths(0, 65536)
    assert lens.sum() == 65536
    assert lens[:-1].min() >= 128 and lens.max() <= 8192
    assert 20 <= len(lens) <= 60
