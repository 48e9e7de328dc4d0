"""Checks that pin the fp64 oracle to facts fixed by the recurrence itself.

The recurrence is the displayed equation of "LT2 transformer looped a tempo lineare"
(section "Sostituire il motore"):  S_t = Diag(a_t)(I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,
read out as o_t = S_t^T q_t.  Every check below compares the oracle with something that is
NOT the oracle's own formula: a closed form that holds for special inputs, an exact
hand-worked example, or an inequality/identity the algebra guarantees.  Each function takes
``lib`` (path of an oracle build, None = the real one) so that the same checks can be run
against copies with a planted mistake.
"""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_examples.json")


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_case(rng, U, L, dk, dv, per_key, s0=True, alpha_lo=0.7):
    q = _unit(rng.standard_normal((U, L, dk)))
    k = _unit(rng.standard_normal((U, L, dk)))
    v = rng.standard_normal((U, L, dv))
    alpha = rng.uniform(alpha_lo, 1.0, size=(U, L, dk) if per_key else (U, L))
    beta = rng.uniform(0.0, 1.0, size=(U, L))
    S0 = rng.standard_normal((U, dk, dv)) if s0 else None
    return q, k, v, alpha, beta, S0


def steps(q, k, v, alpha, beta, S0, per_key, lib=None):
    """All intermediate states S_0..S_L of one head-unit via single-token oracle calls."""
    S = S0.copy()
    out = [S]
    for t in range(q.shape[0]):
        a = alpha[t]
        _, S = oracle.decode_step(q[t], k[t], v[t], a, beta[t], S, per_key=per_key, lib=lib)
        out.append(S)
    return out


# --- P1: alpha = beta = 1 and unit keys make the update an exact overwrite: S_t^T k_t = v_t.
def pin_overwrite(lib=None, seed=1):
    rng = np.random.default_rng(seed)
    U, L, dk, dv = 2, 40, 16, 7
    k = _unit(rng.standard_normal((U, L, dk)))
    v = rng.standard_normal((U, L, dv))
    S0 = rng.standard_normal((U, dk, dv))
    ones = np.ones((U, L))
    # Reading with q = k returns S_t^T k_t, which must equal v_t after each step.
    o, _ = oracle.prefill_sequential(k, k, v, ones, ones, S0=S0, lib=lib)
    err = np.max(np.abs(o - v)) / np.max(np.abs(v))
    assert err < 1e-12, f"overwrite invariant broken: {err}"
    return err


# --- P2: beta = 0 leaves only the decay: S_t = Diag(prod_{s<=t} a_s) S_0, o_t = S_t^T q_t.
def pin_beta_zero(lib=None, per_key=False, seed=2, order="delta_first"):
    rng = np.random.default_rng(seed)
    U, L, dk, dv = 3, 25, 9, 5
    q, k, v, alpha, _, S0 = rand_case(rng, U, L, dk, dv, per_key, alpha_lo=0.5)
    beta = np.zeros((U, L))
    o, S = oracle.prefill_sequential(q, k, v, alpha, beta, S0=S0, per_key=per_key, lib=lib, order=order)
    a = alpha if per_key else np.repeat(alpha[..., None], dk, axis=-1)
    g = np.cumprod(a, axis=1)                                 # [U, L, dk]
    St = g[..., :, None] * S0[:, None, :, :]                  # [U, L, dk, dv]
    o_ref = np.einsum("uld,uldv->ulv", q, St)
    e1 = np.max(np.abs(o - o_ref)) / np.max(np.abs(o_ref))
    e2 = np.max(np.abs(S - St[:, -1])) / np.max(np.abs(St[:, -1]))
    assert max(e1, e2) < 1e-12, f"beta=0 closed form broken: {e1}, {e2}"
    return max(e1, e2)


# --- P3: mutually orthogonal unit keys and S_0 = 0 make every delta term vanish, so the
# mixer is decayed linear attention: o_t = sum_{s<=t} b_s (prod_{s<s'<=t} a_s') (q_t.k_s) v_s.
def pin_orthogonal_keys(lib=None, per_key=False, seed=3, order="delta_first"):
    rng = np.random.default_rng(seed)
    U, dk, dv = 2, 12, 6
    L = dk
    q = rng.standard_normal((U, L, dk))
    v = rng.standard_normal((U, L, dv))
    beta = rng.uniform(0.1, 1.0, size=(U, L))
    if per_key:
        # signed, permuted standard basis: Diag(alpha) keeps these keys orthogonal
        k = np.zeros((U, L, dk))
        idx = np.stack([rng.permutation(dk)[:L] for _ in range(U)])
        sign = rng.choice([-1.0, 1.0], size=(U, L))
        for u in range(U):
            k[u, np.arange(L), idx[u]] = sign[u]
        alpha = rng.uniform(0.5, 1.0, size=(U, L, dk))
    else:
        k = np.stack([np.linalg.qr(rng.standard_normal((dk, dk)))[0].T[:L] for _ in range(U)])
        alpha = rng.uniform(0.5, 1.0, size=(U, L))
    o, _ = oracle.prefill_sequential(q, k, v, alpha, beta, S0=None, per_key=per_key, lib=lib, order=order)
    o_ref = np.zeros_like(o)
    for u in range(U):
        for t in range(L):
            for s in range(t + 1):
                if per_key:
                    i = idx[u, s]
                    dec = np.prod(alpha[u, s + 1:t + 1, i])
                    w = beta[u, s] * dec * q[u, t, i] * k[u, s, i]
                else:
                    dec = np.prod(alpha[u, s + 1:t + 1])
                    w = beta[u, s] * dec * (q[u, t] @ k[u, s])
                o_ref[u, t] += w * v[u, s]
    err = np.max(np.abs(o - o_ref)) / np.max(np.abs(o_ref))
    assert err < 1e-12, f"orthogonal-key closed form broken: {err}"
    return err


# --- P5 and the reading of the gate order: exact hand-worked examples (tests/golden).
def pin_hand_examples(lib=None):
    with open(GOLDEN) as f:
        cases = json.load(f)
    worst = 0.0
    for name, c in cases.items():
        if name.startswith("_"):
            continue
        per_key = c["per_key"]
        q = np.array(c["q"])[None]
        k = np.array(c["k"])[None]
        v = np.array(c["v"])[None]
        alpha = np.array(c["alpha"])[None]
        beta = np.array(c["beta"])[None]
        S0 = np.array(c["S0"])[None]
        o, S = oracle.prefill_sequential(q, k, v, alpha, beta, S0=S0, per_key=per_key, lib=lib)
        e = max(np.max(np.abs(o[0] - np.array(c["o"]))), np.max(np.abs(S[0] - np.array(c["S_L"]))))
        assert e == 0.0, f"hand example {name} differs by {e}"
        worst = max(worst, e)
    return worst


# --- P9: ||A_t||_2 <= max(alpha) <= 1 for beta in [0,1] and ||k|| <= 1, hence
# ||S_t||_F <= ||S_{t-1}||_F + beta_t ||k_t|| ||v_t||.
def pin_non_expansive(lib=None, per_key=False, seed=9):
    rng = np.random.default_rng(seed)
    L, dk, dv = 30, 8, 6
    q, k, v, alpha, beta, S0 = rand_case(rng, 1, L, dk, dv, per_key)
    k = k * rng.uniform(0.3, 1.0, size=(1, L, 1))
    Ss = steps(q[0], k[0], v[0], alpha[0], beta[0], S0[0], per_key, lib=lib)
    for t in range(L):
        lhs = np.linalg.norm(Ss[t + 1])
        rhs = np.linalg.norm(Ss[t]) + beta[0, t] * np.linalg.norm(k[0, t]) * np.linalg.norm(v[0, t])
        assert lhs <= rhs * (1 + 1e-12), f"state grew beyond the bound at t={t}"
    return 0.0


# --- P10 / O8: alpha = beta = 1 with a key that is not exactly unit (as after bf16
# rounding):  S_t^T k - v = (1 - ||k||^2) (S_{t-1}^T k - v)  exactly.
def pin_overwrite_identity(lib=None, seed=10):
    rng = np.random.default_rng(seed)
    L, dk, dv = 20, 10, 4
    k = _unit(rng.standard_normal((L, dk))) * rng.uniform(0.95, 1.05, size=(L, 1))
    v = rng.standard_normal((L, dv))
    S = rng.standard_normal((dk, dv))
    for t in range(L):
        _, S_new = oracle.decode_step(k[t], k[t], v[t], 1.0, 1.0, S, lib=lib)
        lhs = S_new.T @ k[t] - v[t]
        rhs = (1.0 - k[t] @ k[t]) * (S.T @ k[t] - v[t])
        assert np.max(np.abs(lhs - rhs)) < 1e-12 * (1 + np.max(np.abs(S))), "identity broken"
        S = S_new
    return 0.0


# --- P7 (decay-first order, A_t = (I - b_t k_t k_t^T) Diag(a_t)): the delta step acts on the
# already decayed state, so with b = 1 and unit keys the write is an exact overwrite whatever
# the per-key decay: S_t^T k_t = v_t.  (In the printed order the decay comes after the write
# and breaks this as soon as a != 1.)
def pin_overwrite_decay_first(lib=None, seed=11):
    rng = np.random.default_rng(seed)
    U, L, dk, dv = 2, 30, 12, 5
    k = _unit(rng.standard_normal((U, L, dk)))
    v = rng.standard_normal((U, L, dv))
    S0 = rng.standard_normal((U, dk, dv))
    alpha = rng.uniform(0.3, 1.0, size=(U, L, dk))
    ones = np.ones((U, L))
    o, _ = oracle.prefill_sequential(k, k, v, alpha, ones, S0=S0, per_key=True, lib=lib, order="decay_first")
    err = np.max(np.abs(o - v)) / np.max(np.abs(v))
    assert err < 1e-12, f"decay-first overwrite broken: {err}"
    return err


# --- P8: per-key decay equal on every key is scalar gating, for which both orders are the
# same matrix; the decay-first per-key path must then agree with the scalar path.
def pin_uniform_alpha_decay_first(lib=None, seed=12):
    rng = np.random.default_rng(seed)
    U, L, dk, dv = 2, 23, 8, 6
    q, k, v, alpha, beta, S0 = rand_case(rng, U, L, dk, dv, per_key=False, alpha_lo=0.5)
    o_s, S_s = oracle.prefill_sequential(q, k, v, alpha, beta, S0=S0, per_key=False, lib=lib)
    a_vec = np.repeat(alpha[..., None], dk, axis=-1)
    o_d, S_d = oracle.prefill_sequential(q, k, v, a_vec, beta, S0=S0, per_key=True, lib=lib, order="decay_first")
    err = max(np.max(np.abs(o_d - o_s)) / np.max(np.abs(o_s)), np.max(np.abs(S_d - S_s)) / np.max(np.abs(S_s)))
    assert err < 1e-12, f"uniform per-key decay-first differs from scalar gating: {err}"
    return err


ALL_PINS = [
    ("overwrite", lambda lib: pin_overwrite(lib)),
    ("beta_zero", lambda lib: pin_beta_zero(lib, per_key=False)),
    ("beta_zero_per_key", lambda lib: pin_beta_zero(lib, per_key=True)),
    ("orthogonal", lambda lib: pin_orthogonal_keys(lib, per_key=False)),
    ("orthogonal_per_key", lambda lib: pin_orthogonal_keys(lib, per_key=True)),
    ("hand_examples", lambda lib: pin_hand_examples(lib)),
    ("non_expansive", lambda lib: pin_non_expansive(lib, per_key=False)),
    ("non_expansive_per_key", lambda lib: pin_non_expansive(lib, per_key=True)),
    ("overwrite_identity", lambda lib: pin_overwrite_identity(lib)),
    ("overwrite_decay_first", lambda lib: pin_overwrite_decay_first(lib)),
    ("uniform_alpha_decay_first", lambda lib: pin_uniform_alpha_decay_first(lib)),
    ("beta_zero_decay_first", lambda lib: pin_beta_zero(lib, per_key=True, order="decay_first")),
    ("orthogonal_decay_first", lambda lib: pin_orthogonal_keys(lib, per_key=True, order="decay_first")),
]
