"""Pins of the fp64 decode-epilogue oracle ``oracle.gated_rmsnorm``:
per head o / sqrt(mean(o^2) + eps) * weight * silu(z) (flashrt-structures 0.2.0
fused_layer.py ``_decode_one``, rms_norm_gated_silu).  Properties the mathematics fixes,
each also run against copies with a planted mistake, every one of which must fail a pin."""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1)
DV = 16


def pin_scale_invariance(f):
    o = RNG.normal(0, 1, (3, 4, DV))
    z = RNG.normal(0, 1, (3, 4, DV))
    w = RNG.normal(1, 0.2, DV)
    assert np.allclose(f(7.5 * o, z, w, 0.0), f(o, z, w, 0.0), rtol=1e-13, atol=1e-15)


def pin_unit_rms_under_constant_gate(f):
    o = RNG.normal(0, 3, (5, DV))
    c = 1.7
    y = f(o, np.full((5, DV), c), np.ones(DV), 0.0)
    silu_c = c / (1 + math.exp(-c))
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), silu_c, rtol=1e-13)


def pin_silu_values(f):
    o = RNG.normal(0, 1, (4, DV))
    w = np.ones(DV)
    assert np.all(f(o, np.zeros((4, DV)), w, 1e-6) == 0)            # silu(0) = 0
    zp = RNG.normal(0, 2, (4, DV))
    # silu(x) - silu(-x) = x
    assert np.allclose(f(o, zp, w, 0.0) - f(o, -zp, w, 0.0),
                       f(o, np.ones((4, DV)), w, 0.0) / (1 / (1 + math.exp(-1.0))) * zp,
                       rtol=1e-12, atol=1e-14)


def pin_eps_and_zero_input(f):
    z = RNG.normal(0, 1, (2, DV))
    y = f(np.zeros((2, DV)), z, np.ones(DV), 1e-6)
    assert np.all(y == 0)                                           # no NaN at o = 0
    o = np.full((1, DV), 1e-3)
    eps = 1e-6
    y = f(o, np.full((1, DV), 50.0), np.ones(DV), eps)
    assert np.allclose(y, 1e-3 / math.sqrt(1e-6 + eps) * 50.0, rtol=1e-12)


def pin_heads_independent_weight_per_channel(f):
    o = RNG.normal(0, 1, (2, 3, DV))
    z = RNG.normal(0, 1, (2, 3, DV))
    w = RNG.normal(1, 0.3, DV)
    y = f(o, z, w, 1e-5)
    o2 = o.copy()
    o2[:, 1] *= 100.0                                               # one head rescaled
    y2 = f(o2, z, w, 0.0)
    y0 = f(o, z, w, 0.0)
    assert np.allclose(y2[:, 0], y0[:, 0], rtol=1e-13) and np.allclose(y2[:, 2], y0[:, 2], rtol=1e-13)
    yw = f(o, z, np.ones(DV), 1e-5)
    assert np.allclose(y, yw * w, rtol=1e-13, atol=1e-15)           # weight per channel


PINS = [pin_scale_invariance, pin_unit_rms_under_constant_gate, pin_silu_values,
        pin_eps_and_zero_input, pin_heads_independent_weight_per_channel]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_norm_pin(pin):
    pin(oracle.gated_rmsnorm)


def _silu(z):
    return z / (1 + np.exp(-z))


MUTANTS = {
    "sum instead of mean": lambda o, z, w, e: o / np.sqrt(np.sum(o * o, -1, keepdims=True) + e) * w * _silu(z),
    "norm over heads": lambda o, z, w, e: o / np.sqrt(np.mean(o * o, 0, keepdims=True) + e) * w * _silu(z),
    "sigmoid gate": lambda o, z, w, e: o / np.sqrt(np.mean(o * o, -1, keepdims=True) + e) * w / (1 + np.exp(-z)),
    "eps outside sqrt": lambda o, z, w, e: o / (np.sqrt(np.mean(o * o, -1, keepdims=True)) + e) * w * _silu(z),
    "weight ignored": lambda o, z, w, e: o / np.sqrt(np.mean(o * o, -1, keepdims=True) + e) * _silu(z),
    "gate before norm": lambda o, z, w, e: (o * _silu(z)) / np.sqrt(np.mean((o * _silu(z)) ** 2, -1, keepdims=True) + e) * w,
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    caught = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(MUTANTS[name])
        except (AssertionError, FloatingPointError):
            caught += 1
    assert caught > 0, f"mutant '{name}' passes every norm pin"
