"""The fp64 oracle of the sliding-window mixer (oracle/swa.py) against what the definition and
the pages fix (CPU only), and planted mistakes that those checks catch.

"LT2 transformer looped a tempo lineare", section "Sostituire il motore": every token looks at
a window of the w most recent positions; section "Il giro trasforma il calcolo in contesto":
repeated T times, the window reaches back O(T w) tokens.
"""
import math
import types

import numpy as np
import pytest

from oracle import swa


def _case(rng, U=3, L=40, d=8):
    return rng.normal(size=(U, L, d)), rng.normal(size=(U, L, d)), rng.normal(size=(U, L, d))


# ---- pins: each takes the module (or a namespace standing in for it) -------------------------

def pin_window_one_is_identity(f):
    q, k, v = _case(np.random.default_rng(1))
    assert np.allclose(f.prefill(q, k, v, 1), v, atol=1e-15, rtol=0)


def pin_wide_window_is_causal_softmax_attention(f):
    # w >= L: plain causal softmax attention, written here as a running sum over t
    rng = np.random.default_rng(2)
    q, k, v = _case(rng, U=2, L=17, d=5)
    o = f.prefill(q, k, v, 17)
    for u in range(2):
        for t in range(17):
            w = np.exp((k[u, :t + 1] @ q[u, t]) / math.sqrt(5))
            assert np.allclose(o[u, t], (w[:, None] * v[u, :t + 1]).sum(0) / w.sum(), atol=1e-13)


def pin_equal_keys_average_the_window(f):
    # every key equal: uniform weights, o_t = mean of v over the window
    rng = np.random.default_rng(3)
    q, _, v = _case(rng, U=2, L=30, d=4)
    k = np.broadcast_to(rng.normal(size=(2, 1, 4)), (2, 30, 4))
    o = f.prefill(q, k, v, 7)
    for t in range(30):
        assert np.allclose(o[:, t], v[:, max(0, t - 6):t + 1].mean(axis=1), atol=1e-14)


def pin_scale_enters_the_softmax(f):
    # scale 0: uniform weights whatever the keys; a large scale: the arg-max key wins
    rng = np.random.default_rng(4)
    q, k, v = _case(rng, U=1, L=12, d=6)
    o0 = f.prefill(q, k, v, 5, scale=0.0)
    for t in range(12):
        assert np.allclose(o0[0, t], v[0, max(0, t - 4):t + 1].mean(axis=0), atol=1e-14)
    oi = f.prefill(q, k, v, 5, scale=1e4)
    for t in range(12):
        s0 = max(0, t - 4)
        assert np.allclose(oi[0, t], v[0, s0 + np.argmax(k[0, s0:t + 1] @ q[0, t])], atol=1e-9)


def pin_large_scores_stay_finite(f):
    rng = np.random.default_rng(5)
    q, k, v = _case(rng, U=1, L=20, d=4)
    o = f.prefill(q * 300, k * 300, v, 6)
    assert np.isfinite(o).all() and np.all(np.abs(o) <= np.abs(v).max() + 1e-12)


def pin_dense_form_agrees(f):
    rng = np.random.default_rng(6)
    q, k, v = _case(rng, U=3, L=50, d=7)
    for w in (1, 3, 16, 50, 80):
        assert np.allclose(f.prefill(q, k, v, w), swa.prefill_dense(q, k, v, w), atol=1e-13, rtol=0)


def pin_looped_receptive_field(f):
    # T loops chained (each loop's output is the next loop's values, q and k fixed): a change of
    # v at position p reaches exactly the positions t <= p + T (w - 1) -- the pages' O(T w)
    rng = np.random.default_rng(7)
    L, w, T, p = 60, 5, 4, 11
    q, k, v = _case(rng, U=1, L=L, d=6)

    def looped(v0):
        x = v0
        for _ in range(T):
            x = f.prefill(q, k, x, w)
        return x
    d = np.abs(looped(v) - looped(v + np.eye(L)[p][None, :, None])).max(axis=-1)[0]
    assert np.all(d[:p] == 0.0) and np.all(d[p + T * (w - 1) + 1:] == 0.0)
    assert np.all(d[p:p + T * (w - 1) + 1] > 1e-12)


PINS = [pin_window_one_is_identity, pin_wide_window_is_causal_softmax_attention,
        pin_equal_keys_average_the_window, pin_scale_enters_the_softmax, pin_large_scores_stay_finite,
        pin_dense_form_agrees, pin_looped_receptive_field]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(swa)


# ---- planted mistakes: each a variant of the definition that one of the pins must catch -------

def _variant(window_shift=0, include_future=False, no_scale=False, no_max=False):
    def prefill(q, k, v, window, scale=None):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        L, dk = q.shape[-2:]
        sc0 = 1.0 if no_scale else (1.0 / math.sqrt(dk) if scale is None else float(scale))
        qf, kf, vf = q.reshape(-1, L, dk), k.reshape(-1, L, dk), v.reshape(-1, L, v.shape[-1])
        o = np.zeros(vf.shape)
        w = int(window) + window_shift
        for u in range(qf.shape[0]):
            for t in range(L):
                s0 = max(0, t - w + 1)
                s1 = min(L, t + 2) if include_future else t + 1
                sc = sc0 * (kf[u, s0:s1] @ qf[u, t])
                with np.errstate(over="ignore", invalid="ignore"):
                    p = np.exp(sc if no_max else sc - sc.max())
                    o[u, t] = (p / p.sum()) @ vf[u, s0:s1]
        return o.reshape(q.shape[:-2] + (L, v.shape[-1]))
    return types.SimpleNamespace(prefill=prefill)


MUTANTS = {"window one too wide": dict(window_shift=1), "window one too narrow": dict(window_shift=-1),
           "sees the next token": dict(include_future=True), "no 1/sqrt(d) scale": dict(no_scale=True),
           "no max subtraction": dict(no_max=True)}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    f = _variant(**MUTANTS[name])
    caught = 0
    for pin in PINS:
        try:
            pin(f)
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin catches: {name}"
