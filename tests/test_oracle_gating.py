"""Pins of the fp64 gating oracle (``oracle.gating``): g = A softplus(a + dt_bias) with
A = -exp(A_log) per head, beta = beta_scale sigmoid(b) (sparse-delta-memory 2.0.0
sparse_delta_memory/layer.py ``compute_gates``; Rondo-Exp tiny_gdn/fugue.py ``project``).

Each pin is a property the mathematics fixes (special values, identities, asymptotics, the
derivative relation between softplus and sigmoid, per-head broadcasting), and every pin is
also run against copies of the function with a planted mistake, each of which must fail at
least one pin."""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(0)
HV = 5
A = -np.exp(RNG.normal(0.0, 0.5, HV))          # A = -exp(A_log) < 0
DT = RNG.normal(0.0, 1.0, HV)


def pin_special_values(gating):
    a = np.broadcast_to(-DT, (3, HV))          # a + dt_bias = 0 per head
    g, beta = gating(a, np.zeros((3, HV)), A, DT, 1.0)
    assert np.allclose(g, A * math.log(2.0), rtol=1e-15, atol=0)
    assert np.allclose(beta, 0.5, rtol=1e-15, atol=0)


def pin_odd_even_identities(gating):
    x = RNG.normal(0.0, 3.0, (7, HV))
    z = np.zeros(HV)
    gp, bp = gating(x, x, A, z, 1.0)
    gm, bm = gating(-x, -x, A, z, 1.0)
    # softplus(x) - softplus(-x) = x ; sigmoid(x) + sigmoid(-x) = 1
    assert np.allclose(gp - gm, A * x, rtol=1e-12, atol=1e-15)
    assert np.allclose(bp + bm, 1.0, rtol=1e-15, atol=1e-15)


def pin_asymptotics(gating):
    z = np.zeros(HV)
    big = np.full((1, HV), 50.0)
    g, beta = gating(big, big, A, z, 1.0)
    assert np.allclose(g, A * 50.0, rtol=1e-15)               # softplus(x) -> x
    assert np.allclose(beta, 1.0, rtol=0, atol=1e-20)         # sigmoid(x) -> 1
    g, beta = gating(-big, -big, A, z, 1.0)
    assert np.allclose(g, A * math.exp(-50.0), rtol=1e-12)    # softplus(x) -> e^x
    assert np.allclose(beta, math.exp(-50.0), rtol=1e-12)     # sigmoid(x) -> e^x


def pin_derivative(gating):
    """d/da softplus(a + dt) = sigmoid(a + dt): the two halves agree with each other."""
    a = RNG.normal(0.0, 2.0, (6, HV))
    h = 1e-6
    gp, _ = gating(a + h, a, A, DT, 1.0)
    gm, _ = gating(a - h, a, A, DT, 1.0)
    _, sig = gating(a, a + DT, A, DT, 1.0)
    assert np.allclose((gp - gm) / (2 * h), A * sig, rtol=1e-7, atol=1e-9)


def pin_decay_range_and_scale(gating):
    a = RNG.normal(-2.0, 1.0, (9, HV))
    b = RNG.normal(0.0, 1.0, (9, HV))
    g, beta1 = gating(a, b, A, DT, 1.0)
    _, beta2 = gating(a, b, A, DT, 2.0)
    assert np.all(g < 0) and np.all(np.exp(g) > 0) and np.all(np.exp(g) < 1)
    assert np.all((beta1 > 0) & (beta1 < 1))
    assert np.allclose(beta2, 2.0 * beta1, rtol=1e-15, atol=0)
    g0, _ = gating(a, b, np.zeros(HV), DT, 1.0)               # A = 0: no decay, alpha = 1
    assert np.all(g0 == 0)


def pin_per_head_parameters(gating):
    """A and dt_bias index the last (head) axis, whatever the leading shape."""
    a = RNG.normal(0.0, 1.0, (2, 3, HV))
    g, _ = gating(a, a, A, DT, 1.0)
    for h in range(HV):
        gh, _ = gating(a[..., h:h + 1], a[..., h:h + 1], A[h:h + 1], DT[h:h + 1], 1.0)
        assert np.allclose(g[..., h:h + 1], gh, rtol=1e-15, atol=0)
    gs, _ = gating(np.broadcast_to(-DT, (2, 3, HV)), a, A, DT, 1.0)
    assert np.allclose(gs, A * math.log(2.0), rtol=1e-15)


PINS = [pin_special_values, pin_odd_even_identities, pin_asymptotics, pin_derivative,
        pin_decay_range_and_scale, pin_per_head_parameters]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_gating_pin(pin):
    pin(oracle.gating)


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return np.exp(-np.logaddexp(0.0, -x))


MUTANTS = {
    "no dt_bias": lambda a, b, A, dt, s=1.0: (A * _softplus(np.asarray(a, float)), s * _sigmoid(np.asarray(b, float))),
    "sign of A": lambda a, b, A, dt, s=1.0: (-A * _softplus(a + dt), s * _sigmoid(np.asarray(b, float))),
    "sigmoid(-b)": lambda a, b, A, dt, s=1.0: (A * _softplus(a + dt), s * _sigmoid(-np.asarray(b, float))),
    "exp for softplus": lambda a, b, A, dt, s=1.0: (A * np.exp(a + dt), s * _sigmoid(np.asarray(b, float))),
    "beta_scale ignored": lambda a, b, A, dt, s=1.0: (A * _softplus(a + dt), _sigmoid(np.asarray(b, float))),
    "dt_bias outside softplus": lambda a, b, A, dt, s=1.0: (A * (_softplus(np.asarray(a, float)) + dt), s * _sigmoid(np.asarray(b, float))),
    "log1p(x) for softplus": lambda a, b, A, dt, s=1.0: (A * np.log1p(np.abs(a + dt)), s * _sigmoid(np.asarray(b, float))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    mutant = MUTANTS[name]
    caught = 0
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught += 1
    assert caught > 0, f"mutant '{name}' passes every gating pin"
