"""The backward-pass oracle (oracle/backward.py) against central finite differences of the
forward oracle (the compiled sequential one, a separate code path), CPU only, and planted
mistakes that the check catches.

"LT2 transformer looped a tempo lineare", section "Sostituire il motore", displayed equation: the
gradients are those of loss = sum(dO * o) + sum(dS_L * S_L) through the recurrence.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import backward as obw

EPS = 1e-6


def _case(rng, per_key, U=2, L=7, dk=4, dv=3):
    q = rng.normal(size=(U, L, dk))
    k = rng.normal(size=(U, L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(U, L, dv))
    alpha = rng.uniform(0.5, 1.0, size=(U, L, dk) if per_key else (U, L))
    beta = rng.uniform(0.05, 0.95, size=(U, L))
    S0 = rng.normal(size=(U, dk, dv))
    dO = rng.normal(size=(U, L, dv))
    dSL = rng.normal(size=(U, dk, dv))
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0), dO, dSL


def _loss(x, dO, dSL, per_key, order):
    o, S = oracle.prefill_sequential(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x["S0"], per_key=per_key,
                                     order=order)
    return float(np.sum(dO * o) + np.sum(dSL * S))


def pin_matches_finite_differences(f, per_key, order, seed=0):
    rng = np.random.default_rng(seed)
    x, dO, dSL = _case(rng, per_key)
    g = f.backward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], dO, S0=x["S0"], dS_L=dSL, per_key=per_key,
                   order=order)
    names = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "beta": "dbeta", "S0": "dS0"}
    for n, gn in names.items():
        for trial in range(2):
            d = rng.normal(size=x[n].shape)
            xp = dict(x)
            xm = dict(x)
            xp[n] = x[n] + EPS * d
            xm[n] = x[n] - EPS * d
            fd = (_loss(xp, dO, dSL, per_key, order) - _loss(xm, dO, dSL, per_key, order)) / (2 * EPS)
            an = float(np.sum(g[gn] * d))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (n, trial, fd, an)


VARIANTS = [(False, "delta_first"), (True, "delta_first"), (True, "decay_first")]


@pytest.mark.parametrize("per_key,order", VARIANTS)
def test_gradients_match_finite_differences(per_key, order):
    pin_matches_finite_differences(obw, per_key, order)


def test_no_upstream_gradient_gives_zero():
    rng = np.random.default_rng(1)
    x, dO, _ = _case(rng, False)
    g = obw.backward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], np.zeros_like(dO), S0=x["S0"])
    assert all(np.all(t == 0) for t in g.values())


def test_readout_only_gradient_closed_form():
    # dO only at the last token, dS_L = 0: dq_L = S_L dO_L, and dv_L = beta_L (q_L . k_L) dO_L
    # (o_L = S_L^T q_L with S_L holding beta_L k_L v_L^T as its only v_L term)
    rng = np.random.default_rng(2)
    x, dO, _ = _case(rng, False)
    dO[:] = 0.0
    dO[:, -1] = rng.normal(size=dO[:, -1].shape)
    g = obw.backward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], dO, S0=x["S0"])
    _, S = oracle.prefill_sequential(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x["S0"])
    for u in range(2):
        assert np.allclose(g["dq"][u, -1], S[u] @ dO[u, -1], atol=1e-13)
        qk = x["q"][u, -1] @ x["k"][u, -1]
        assert np.allclose(g["dv"][u, -1], x["beta"][u, -1] * qk * dO[u, -1], atol=1e-13)


# ---- planted mistakes: each changes one gradient the way a slip in the derivation would --------

def _mutant(change):
    def backward(*a, **kw):
        g = obw.backward(*a, **kw)
        change(g)
        return g
    return types.SimpleNamespace(backward=backward)


def _drop_last_token_dk(g):
    g["dk"][..., -1, :] = 0.0


def _dalpha_scaled(g):
    g["dalpha"] *= 1.001


def _dS0_rows_reversed(g):
    g["dS0"] = g["dS0"][..., ::-1, :].copy()


def _dbeta_sign(g):
    g["dbeta"][..., 0] *= -1.0


MUTANTS = {"dk of the last token dropped": _drop_last_token_dk, "dalpha off by 0.1 %": _dalpha_scaled,
           "dS0 rows permuted": _dS0_rows_reversed, "dbeta of the first token negated": _dbeta_sign}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    f = _mutant(MUTANTS[name])
    with pytest.raises(AssertionError):
        for per_key, order in VARIANTS:
            pin_matches_finite_differences(f, per_key, order, seed=3)
