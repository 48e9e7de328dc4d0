"""The fp64 oracle of the fused prologue and epilogue (oracle/fused.py) against values the
definitions fix (CPU only), and planted mistakes that those checks catch.

Prologue: q, k normalised to unit L2 norm per (token, head); beta = sigmoid(b);
alpha = exp(-softplus(a) c).  Epilogue: o <- sigmoid(z) o (the output gate of "LT2 transformer
looped a tempo lineare", section "Dove il quadro si incrina").
"""
import math
import types

import numpy as np
import pytest

from oracle import fused


# ---- pins: each takes the module (or a namespace standing in for it) -------------------------

def pin_l2(f):
    assert np.array_equal(f.l2_normalize(np.array([3.0, 4.0])), np.array([0.6, 0.8]))
    rng = np.random.default_rng(3)
    x = rng.normal(size=(50, 7)) * rng.uniform(0.01, 100, size=(50, 1))
    y = f.l2_normalize(x)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-15, rtol=0)
    assert np.allclose(np.sum(x * y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14, atol=0)
    assert np.allclose(f.l2_normalize(5.0 * x), y, atol=1e-15, rtol=0)
    assert np.array_equal(f.l2_normalize(np.zeros((2, 4))), np.zeros((2, 4)))


def pin_sigmoid(f):
    assert f.sigmoid(0.0) == 0.5
    assert abs(f.sigmoid(math.log(3.0)) - 0.75) < 1e-16
    assert abs(f.sigmoid(-math.log(3.0)) - 0.25) < 1e-16
    x = np.linspace(-30, 30, 121)
    assert np.allclose(f.sigmoid(x) + f.sigmoid(-x), 1.0, atol=1e-15, rtol=0)
    assert f.sigmoid(1000.0) == 1.0 and 0.0 <= f.sigmoid(-1000.0) < 1e-300


def pin_softplus(f):
    assert abs(f.softplus(0.0) - math.log(2.0)) < 1e-16
    assert abs(f.softplus(math.log(3.0)) - math.log(4.0)) < 1e-15
    x = np.linspace(-30, 30, 121)
    assert np.allclose(f.softplus(x) - f.softplus(-x), x, atol=1e-13, rtol=0)
    assert f.softplus(1000.0) == 1000.0


def pin_alpha(f):
    # exp(-softplus(a)) = 1 / (1 + e^a), so alpha(ln 3, 1) = 1/4; alpha(0, c) = 2^-c
    assert abs(f.gate_alpha(math.log(3.0), 1.0) - 0.25) < 1e-16
    assert abs(f.gate_alpha(0.0, 0.1) - 2.0 ** -0.1) < 1e-16
    a = np.linspace(-20, 20, 81)
    al = f.gate_alpha(a, 0.1)
    assert np.all(np.diff(al) < 0) and np.all((al > 0) & (al <= 1))
    assert f.gate_alpha(-800.0, 0.1) == 1.0


def pin_output_gate(f):
    o = np.array([2.0, -6.0, 1.5])
    assert np.array_equal(f.output_gate(o, np.zeros(3)), o / 2)
    assert np.allclose(f.output_gate(o, np.full(3, math.log(3.0))), 0.75 * o, atol=1e-15, rtol=0)
    assert np.array_equal(f.output_gate(o, np.full(3, 1000.0)), o)


def pin_overwrite_through_the_prologue(f):
    # raw keys of any norm, beta logits -> +inf (beta = 1), alpha logits -> -inf (alpha = 1):
    # after the prologue every token overwrites its own key's value, so with q = k the readout
    # is v_t (the overwrite property of the recurrence), and the output gate with z = 0 halves it
    rng = np.random.default_rng(7)
    L, dk, dv = 9, 5, 4
    k = rng.normal(size=(2, L, dk)) * rng.uniform(0.1, 10, size=(2, L, 1))
    v = rng.normal(size=(2, L, dv))
    a = np.full((2, L), -800.0)
    b = np.full((2, L), 800.0)
    o, _ = f.prefill(k, k, v, a, b, z=np.zeros((2, L, dv)), S0=rng.normal(size=(2, dk, dv)),
                     alpha_scale=0.1)
    assert np.allclose(o, v / 2, atol=1e-12, rtol=0)


PINS = [pin_l2, pin_sigmoid, pin_softplus, pin_alpha, pin_output_gate, pin_overwrite_through_the_prologue]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(fused)


# ---- planted mistakes -------------------------------------------------------------------------

def _mutant(**over):
    """The oracle's functions with some replaced; prefill re-composed from this namespace."""
    ns = types.SimpleNamespace(**{n: getattr(fused, n) for n in
                                  ("l2_normalize", "sigmoid", "softplus", "gate_alpha", "gate_beta",
                                   "output_gate")})
    for n, fn in over.items():
        setattr(ns, n, fn)

    def prefill(q, k, v, a, b, z=None, S0=None, per_key=False, order="delta_first", qk_l2norm=True,
                gate_logits=True, alpha_scale=1.0):
        qn, kn = (ns.l2_normalize(q), ns.l2_normalize(k)) if qk_l2norm else (q, k)
        al, be = (ns.gate_alpha(a, alpha_scale), ns.gate_beta(b)) if gate_logits else (a, b)
        o, S = fused.prefill_sequential(qn, kn, v, al, be, S0=S0, per_key=per_key, order=order)
        return (o if z is None else ns.output_gate(o, z)), S
    ns.prefill = prefill
    return ns


def _sig_flipped(x):
    return 1.0 / (1.0 + np.exp(np.asarray(x, dtype=np.float64)))


MUTANTS = {
    "norm without the square root": dict(l2_normalize=lambda x, eps=1e-12: np.asarray(x, float) / np.maximum(
        np.sum(np.asarray(x, float) ** 2, axis=-1, keepdims=True), eps)),
    "sigmoid of -x": dict(sigmoid=_sig_flipped),
    "softplus as exp": dict(softplus=lambda x: np.exp(np.asarray(x, float))),
    "alpha scale ignored": dict(gate_alpha=lambda a, c: np.exp(-fused.softplus(a))),
    "alpha without the minus": dict(gate_alpha=lambda a, c: np.exp(fused.softplus(a) * c)),
    "beta not squashed": dict(gate_beta=lambda b: np.asarray(b, float)),
    "gate multiplies by z": dict(output_gate=lambda o, z: np.asarray(z, float) * np.asarray(o, float)),
    "gate of 1 - sigmoid": dict(output_gate=lambda o, z: (1 - fused.sigmoid(z)) * np.asarray(o, float)),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    ns = _mutant(**MUTANTS[name])
    caught = 0
    for pin in PINS:
        try:
            pin(ns)
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught > 0, f"no pin catches: {name}"
