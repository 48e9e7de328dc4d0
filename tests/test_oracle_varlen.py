"""The packed-sequence oracle (oracle/varlen.py) against what the definition fixes (CPU only),
and planted mistakes that those checks catch.

"LT2 transformer looped a tempo lineare", section "Sostituire il motore", displayed equation: a
sequence's recurrence starts from its own initial state and reads only its own tokens.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import varlen


def _packed(rng, lens, T=2, H=2, d=8):
    N = int(sum(lens))
    q = rng.normal(size=(T, H, N, d))
    k = rng.normal(size=(T, H, N, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, N, d))
    alpha = rng.uniform(0.8, 1.0, size=(T, H, N))
    beta = rng.uniform(0.0, 1.0, size=(T, H, N))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0 = rng.normal(size=(T, len(lens), H, d, d))
    return q, k, v, alpha, beta, cu, S0


# ---- pins: each takes the module (or a namespace standing in for it) -------------------------

def pin_equal_lengths_match_the_fixed_layout(f):
    # B sequences of one length L packed along the token axis are the fixed [T, B, H, L] layout
    rng = np.random.default_rng(1)
    T, B, H, L, d = 2, 3, 2, 9, 6
    q, k, v, al, be, cu, S0 = _packed(rng, [L] * B, T, H, d)
    o, S = f.prefill(q, k, v, al, be, cu, S0=S0)
    unpack = lambda x: x.reshape(T, H, B, L, *x.shape[3:]).swapaxes(1, 2)   # [T, B, H, L, ...]
    o_ref, S_ref = oracle.prefill_sequential(unpack(q), unpack(k), unpack(v), unpack(al), unpack(be), S0=S0)
    assert np.allclose(unpack(o), o_ref, atol=1e-13, rtol=0) and np.allclose(S, S_ref, atol=1e-13, rtol=0)


def pin_sequences_are_independent(f):
    # changing every input of sequence 1 leaves sequences 0 and 2 bit-identical
    rng = np.random.default_rng(2)
    lens = [5, 7, 4]
    q, k, v, al, be, cu, S0 = _packed(rng, lens)
    o1, S1 = f.prefill(q, k, v, al, be, cu, S0=S0)
    q2, v2, S02 = q.copy(), v.copy(), S0.copy()
    q2[:, :, cu[1]:cu[2]] *= -1.0
    v2[:, :, cu[1]:cu[2]] += 3.0
    S02[:, 1] += 1.0
    o2, S2 = f.prefill(q2, k, v2, al, be, cu, S0=S02)
    for b in (0, 2):
        assert np.array_equal(o1[:, :, cu[b]:cu[b + 1]], o2[:, :, cu[b]:cu[b + 1]])
        assert np.array_equal(S1[:, b], S2[:, b])
    assert not np.array_equal(S1[:, 1], S2[:, 1])


def pin_pure_decay_from_each_own_state(f):
    # beta = 0: S_end = prod(alpha) S0_b and o_t = S_t^T q_t with S_t = prod_{s<=t} alpha_s S0_b,
    # per sequence from its own S0 (a closed form of the recurrence)
    rng = np.random.default_rng(3)
    lens = [3, 6, 1, 4]
    q, k, v, al, _, cu, S0 = _packed(rng, lens)
    be = np.zeros(al.shape)
    o, S = f.prefill(q, k, v, al, be, cu, S0=S0)
    for b in range(len(lens)):
        g = np.cumprod(al[:, :, cu[b]:cu[b + 1]], axis=-1)                     # [T, H, n]
        o_ref = np.einsum("thn,thij,thni->thnj", g, S0[:, b], q[:, :, cu[b]:cu[b + 1]])
        assert np.allclose(o[:, :, cu[b]:cu[b + 1]], o_ref, atol=1e-13)
        assert np.allclose(S[:, b], g[..., -1][..., None, None] * S0[:, b], atol=1e-13)


def pin_empty_sequence_passes_its_state(f):
    rng = np.random.default_rng(4)
    q, k, v, al, be, cu, S0 = _packed(rng, [4, 0, 5])
    o, S = f.prefill(q, k, v, al, be, cu, S0=S0)
    assert np.array_equal(S[:, 1], S0[:, 1]) and o.shape[2] == 9
    _, S_zero = f.prefill(q, k, v, al, be, cu, S0=None)
    assert np.array_equal(S_zero[:, 1], np.zeros_like(S_zero[:, 1]))


PINS = [pin_equal_lengths_match_the_fixed_layout, pin_sequences_are_independent,
        pin_pure_decay_from_each_own_state, pin_empty_sequence_passes_its_state]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(varlen)


def test_fused_form_slices_the_same_way():
    # raw inputs through the fused oracle, per sequence, equal the fused oracle on each slice
    from oracle import fused
    rng = np.random.default_rng(5)
    lens = [6, 3]
    T, H, d = 2, 2, 8
    N = sum(lens)
    q, k, v, z = (rng.normal(size=(T, H, N, d)) for _ in range(4))
    a, b = rng.normal(size=(T, H, N)), rng.normal(size=(T, H, N))
    cu = np.array([0, 6, 9])
    o, S = varlen.prefill(q, k, v, a, b, cu, raw=dict(z=z, alpha_scale=0.1))
    for i in range(2):
        sl = slice(cu[i], cu[i + 1])
        ob, Sb = fused.prefill(q[:, :, sl], k[:, :, sl], v[:, :, sl], a[:, :, sl], b[:, :, sl], z=z[:, :, sl],
                               alpha_scale=0.1)
        assert np.allclose(o[:, :, sl], ob, atol=1e-14) and np.allclose(S[:, i], Sb, atol=1e-14)


# ---- planted mistakes -------------------------------------------------------------------------

def _variant(carry_state=False, shift=0, s0_from_previous=False):
    def prefill(q, k, v, alpha, beta, cu_seqlens, S0=None, per_key=False, order="delta_first", raw=None):
        T, H, N, dk = q.shape
        dv = v.shape[-1]
        cu = [int(c) for c in cu_seqlens]
        B = len(cu) - 1
        o = np.zeros((T, H, N, dv))
        S = np.zeros((T, B, H, dk, dv))
        prev = None
        for b in range(B):
            c0, c1 = min(cu[b] + shift, cu[b + 1]), cu[b + 1]
            s0 = None if S0 is None else S0[:, (b - 1) % B if s0_from_previous else b]
            if carry_state and prev is not None:
                s0 = prev
            if c1 == c0:
                S[:, b] = 0.0 if s0 is None else s0
                prev = S[:, b]
                continue
            sl = slice(c0, c1)
            ob, Sb = oracle.prefill_sequential(q[:, :, sl], k[:, :, sl], v[:, :, sl], alpha[:, :, sl],
                                               beta[:, :, sl], S0=s0)
            o[:, :, sl] = ob
            S[:, b] = Sb
            prev = Sb
        return o, S
    return types.SimpleNamespace(prefill=prefill)


MUTANTS = {"state carried across sequences": dict(carry_state=True),
           "offsets off by one": dict(shift=1),
           "initial state of the wrong sequence": dict(s0_from_previous=True)}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    f = _variant(**MUTANTS[name])
    caught = 0
    for pin in PINS:
        try:
            pin(f)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin catches: {name}"
