"""Pins for the prologue oracle (oracle/prologue.py) from closed forms: a 3-4-5
vector, unit norms and scale invariance for the L2 normalisation; alpha(0) = 1/2,
alpha(ln(e - 1)) = 1/e, alpha(x) / alpha(-x) = e^-x and the tails (alpha(40) ~ e^-40,
1 - alpha(-20) ~ e^-20) for the gate.
Planted mistakes must fail them."""

import math

import numpy as np
import pytest

from oracle import apply_prologue, gate_from_logit, l2_normalise


def pins_norm(norm):
    ok = np.allclose(norm(np.array([3.0, 4.0])), [0.6, 0.8], rtol=0, atol=1e-7)
    ok &= np.array_equal(norm(np.zeros(5)), np.zeros(5))
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 128)) * rng.uniform(0.1, 10, size=(7, 1))
    n = norm(x)
    ok &= np.allclose(np.linalg.norm(n, axis=-1), 1.0, atol=1e-6)
    ok &= np.allclose(norm(5.0 * x), n, atol=1e-7)
    ok &= np.allclose(n / np.linalg.norm(n, axis=-1, keepdims=True),
                      x / np.linalg.norm(x, axis=-1, keepdims=True), atol=1e-12)
    return bool(ok)


def pins_gate(gate):
    ok = abs(gate(0.0) - 0.5) < 1e-15
    ok &= abs(gate(math.log(math.e - 1.0)) - math.exp(-1.0)) < 1e-15
    x = np.linspace(-20, 20, 81)
    ok &= np.allclose(gate(x) / gate(-x), np.exp(-x), rtol=1e-12)
    ok &= abs(gate(40.0) / math.exp(-40.0) - 1.0) < 1e-12
    ok &= abs((1.0 - gate(-20.0)) / math.exp(-20.0) - 1.0) < 1e-6
    ok &= bool(np.all(np.diff(gate(x)) < 0)) and bool(np.all((gate(x) > 0) & (gate(x) < 1)))
    return bool(ok)


def test_normalisation_pins():
    assert pins_norm(l2_normalise)


def test_gate_pins():
    assert pins_gate(gate_from_logit)


MUTANT_NORMS = {
    "no_sqrt": lambda x: np.asarray(x, float) / ((np.asarray(x, float) ** 2).sum(-1, keepdims=True) + 1e-6),
    "l1": lambda x: np.asarray(x, float) / (np.abs(np.asarray(x, float)).sum(-1, keepdims=True) + 1e-6),
    "eps_outside_large": lambda x: np.asarray(x, float) / (np.sqrt((np.asarray(x, float) ** 2).sum(-1, keepdims=True)) + 1e-2),
}
MUTANT_GATES = {
    "plus_softplus": lambda x: np.exp(np.log1p(np.exp(np.asarray(x, float)))),
    "sigmoid": lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, float))),
    "exp_minus_x": lambda x: np.exp(-np.asarray(x, float)),
}


@pytest.mark.parametrize("kind", sorted(MUTANT_NORMS))
def test_norm_pins_catch_planted_mistake(kind):
    assert not pins_norm(MUTANT_NORMS[kind])


@pytest.mark.parametrize("kind", sorted(MUTANT_GATES))
def test_gate_pins_catch_planted_mistake(kind):
    with np.errstate(over="ignore"):
        assert not pins_gate(MUTANT_GATES[kind])


def test_flags_pass_tensors_through():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((2, 3, 8)), rng.standard_normal((2, 3, 8))
    a = rng.uniform(0.1, 0.9, size=(2, 3))
    q2, k2, a2 = apply_prologue(q, k, a, l2norm=False, gate_logit=False)
    assert np.array_equal(q2, q) and np.array_equal(k2, k) and np.array_equal(a2, a)


def test_bf16_rounding_is_nearest():
    """The bf16 cast of the normalised vectors: every value lands within half a bf16
    unit (2^-8 relative: 8 significant bits) and on a bf16 grid point."""
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 64))
    q2, _, _ = apply_prologue(q, q, np.zeros(4), gate_logit=False, bf16=True)
    exact = l2_normalise(q)
    assert np.all(np.abs(q2 - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-30)
    bits = q2.astype(np.float32).view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
