"""The fp64 oracle against facts the recurrence fixes (CPU only).

Recurrence: "LT2 transformer looped a tempo lineare", section "Sostituire il motore",
displayed equation.  Loops are independent recurrences (section "Dove il quadro si incrina":
carrying state across loops is listed as unexplored).
"""
import numpy as np
import pytest

import oracle
from oracle import twin
from tests import oracle_pins as pins
from tests.oracle_pins import rand_case


@pytest.mark.parametrize("name,check", pins.ALL_PINS, ids=[n for n, _ in pins.ALL_PINS])
def test_pin(name, check):
    check(None)


@pytest.mark.parametrize("per_key,order", [(False, "delta_first"), (True, "delta_first"), (True, "decay_first")])
def test_sequential_dense_twin_agree(per_key, order):
    # c2: the transition matrix built densely (C code and an independent numpy twin).
    rng = np.random.default_rng(11)
    q, k, v, a, b, S0 = rand_case(rng, 3, 13, 6, 5, per_key)
    o1, S1 = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=per_key, order=order)
    o2, S2 = oracle.prefill_dense(q, k, v, a, b, S0=S0, per_key=per_key, order=order)
    o3, S3 = twin.prefill(q, k, v, a, b, S0=S0, per_key=per_key, order=order)
    for x, y in ((o2, o1), (S2, S1), (o3, o1), (S3, S1)):
        assert np.max(np.abs(x - y)) <= 1e-13 * max(1.0, np.max(np.abs(y)))


@pytest.mark.parametrize("C", [1, 2, 8, 16, 64])
@pytest.mark.parametrize("L", [1, 5, 63, 64, 65, 200])
@pytest.mark.parametrize("per_key,form,order", [(False, "u", "delta_first"), (False, "e", "delta_first"),
                                                (False, "wy", "delta_first"),
                                                (True, "e", "delta_first"), (True, "e", "decay_first")])
def test_chunked_equals_sequential(C, L, per_key, form, order):
    # P4: the chunk-parallel rewriting used by the GPU equals the token-by-token equation.
    rng = np.random.default_rng(1000 + C + 7 * L + (13 if per_key else 0))
    q, k, v, a, b, S0 = rand_case(rng, 2, L, 8, 5, per_key)
    o1, S1 = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=per_key, order=order)
    o2, S2 = oracle.prefill_chunked(q, k, v, a, b, S0=S0, per_key=per_key, chunk=C, form=form, order=order)
    assert oracle.rel_max_err(o2, o1) < 1e-12
    assert oracle.rel_max_err(S2, S1) < 1e-12


def test_chunked_strong_decay():
    # Chunk-local decay products as small as ~1e-40 stay exact in fp64.
    rng = np.random.default_rng(5)
    q, k, v, a, b, S0 = rand_case(rng, 1, 130, 8, 4, True, alpha_lo=0.2)
    o1, S1 = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=True)
    o2, S2 = oracle.prefill_chunked(q, k, v, a, b, S0=S0, per_key=True, chunk=64, form="e")
    assert oracle.rel_max_err(o2, o1) < 1e-12 and oracle.rel_max_err(S2, S1) < 1e-12


@pytest.mark.parametrize("per_key", [False, True])
def test_segment_resume(per_key):
    # P6: prefill(L1 + L2) == prefill(L2, S0 = S_{L1}) after prefill(L1).
    rng = np.random.default_rng(6)
    q, k, v, a, b, S0 = rand_case(rng, 2, 50, 7, 3, per_key)
    o, S = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=per_key)
    oa, Sa = oracle.prefill_sequential(q[:, :21], k[:, :21], v[:, :21], a[:, :21], b[:, :21],
                                       S0=S0, per_key=per_key)
    ob, Sb = oracle.prefill_sequential(q[:, 21:], k[:, 21:], v[:, 21:], a[:, 21:], b[:, 21:],
                                       S0=Sa, per_key=per_key)
    assert np.max(np.abs(np.concatenate([oa, ob], axis=1) - o)) < 1e-13
    assert np.max(np.abs(Sb - S)) < 1e-13


@pytest.mark.parametrize("per_key", [False, True])
def test_decode_stepped_equals_prefill(per_key):
    # P7: L single-token steps reproduce the prefill.
    rng = np.random.default_rng(7)
    q, k, v, a, b, S0 = rand_case(rng, 3, 17, 5, 4, per_key)
    o, S = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=per_key)
    St = S0
    for t in range(q.shape[1]):
        ot, St = oracle.decode_step(q[:, t], k[:, t], v[:, t], a[:, t], b[:, t], St,
                                    per_key=per_key)
        assert np.max(np.abs(ot - o[:, t])) < 1e-13
    assert np.max(np.abs(St - S)) < 1e-13


def test_loop_independence_and_permutation():
    # P8: slicing the [T,B,H] result at loop tau equals a call on that slice alone, and
    # permuting (b, h) permutes the outputs.
    rng = np.random.default_rng(8)
    T, B, H, L, d = 3, 2, 2, 9, 4
    q, k, v, a, b, S0 = rand_case(rng, T * B * H, L, d, d, False)
    rs = lambda x: x.reshape((T, B, H) + x.shape[1:])
    q, k, v, a, b, S0 = map(rs, (q, k, v, a, b, S0))
    o, S = oracle.prefill_sequential(q, k, v, a, b, S0=S0)
    for tau in range(T):
        ot, St = oracle.prefill_sequential(q[tau], k[tau], v[tau], a[tau], b[tau], S0=S0[tau])
        assert np.array_equal(ot, o[tau]) and np.array_equal(St, S[tau])
    perm_b, perm_h = [1, 0], [1, 0]
    P = lambda x: x[:, perm_b][:, :, perm_h]
    op, Sp = oracle.prefill_sequential(P(q), P(k), P(v), P(a), P(b), S0=P(S0))
    assert np.array_equal(op, P(o)) and np.array_equal(Sp, P(S))


def test_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(12)
    q, k, v, a, b, S0 = rand_case(rng, 2, 0, 4, 3, False)
    o, S = oracle.prefill_sequential(q, k, v, a, b, S0=S0)
    assert o.shape == (2, 0, 3) and np.array_equal(S, S0)


def test_parity_metric():
    ref = np.array([3.0, -4.0])          # rms = sqrt(12.5)
    assert abs(oracle.rel_max_err(ref + [0.5, 0.0], ref) - 0.5 / np.sqrt(12.5)) < 1e-15


def test_orders_differ_per_key_and_agree_for_scalar_decay():
    # The two readings of the per-key equation are different recurrences (so the pins above
    # tell them apart), except when the decay is the same on every key.
    rng = np.random.default_rng(13)
    q, k, v, a, b, S0 = rand_case(rng, 2, 17, 6, 4, True, alpha_lo=0.5)
    o1, _ = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=True)
    o2, _ = oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=True, order="decay_first")
    assert oracle.rel_max_err(o2, o1) > 1e-2
    a1 = np.repeat(a[..., :1], 6, axis=-1)
    o1, _ = oracle.prefill_sequential(q, k, v, a1, b, S0=S0, per_key=True)
    o2, _ = oracle.prefill_sequential(q, k, v, a1, b, S0=S0, per_key=True, order="decay_first")
    assert oracle.rel_max_err(o2, o1) < 1e-13
    with pytest.raises(ValueError):
        oracle.prefill_sequential(q, k, v, a, b, S0=S0, per_key=True, order="sideways")
