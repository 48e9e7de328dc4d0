"""fp64 oracle of the steps fused on either side of the mixer (test infrastructure only).

The product path never imports this module.  Everything is plain numpy in float64, written from
the definitions:

Prologue (the input recipe of the workloads, "LT2 transformer looped a tempo lineare", section
"Sostituire il motore": the gated delta rule takes unit-norm keys and queries, a write strength
beta in (0, 1) and a decay alpha in (0, 1]):
    q^ = q / max(||q||_2, eps),  k^ = k / max(||k||_2, eps)      per (token, head), over d_k
    beta = sigmoid(b) = 1 / (1 + e^{-b})
    alpha = exp(-softplus(a) * c),  softplus(a) = log(1 + e^a)    (scalar, or per key channel)

Epilogue (the sigmoid output gate of the same page, section "Dove il quadro si incrina", which
keeps the state norm in check inside the loop; the wispaper.ai blog, section "Critical Insight:
The Attention Sink Mitigation", names it an SDPA output gate):
    o <- sigmoid(z) (.) o        z given per (token, head, value channel)

Between them runs the recurrence itself, through the sequential oracle of ``oracle``.
"""
import numpy as np

from . import decode_step, prefill_sequential

L2_EPS = 1e-12


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def l2_normalize(x, eps=L2_EPS):
    """x / max(||x||_2, eps) over the last axis (a zero row stays zero)."""
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def sigmoid(x):
    """1 / (1 + e^{-x}), evaluated without overflow for either sign of x."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def softplus(x):
    """log(1 + e^x) = max(x, 0) + log(1 + e^{-|x|})."""
    x = _f64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def gate_beta(b):
    return sigmoid(b)


def gate_alpha(a, c):
    return np.exp(-softplus(a) * float(c))


def output_gate(o, z):
    return sigmoid(z) * _f64(o)


def prologue(q, k, a, b, qk_l2norm=True, gate_logits=True, alpha_scale=1.0):
    """The recurrence's inputs from the raw ones: (q^, k^, alpha, beta)."""
    if qk_l2norm:
        q, k = l2_normalize(q), l2_normalize(k)
    if gate_logits:
        return _f64(q), _f64(k), gate_alpha(a, alpha_scale), gate_beta(b)
    return _f64(q), _f64(k), _f64(a), _f64(b)


def prefill(q, k, v, a, b, z=None, S0=None, per_key=False, order="delta_first", qk_l2norm=True,
            gate_logits=True, alpha_scale=1.0):
    """Prologue, the looped recurrence over all tokens, epilogue.  Returns (o, S_L) in fp64."""
    qn, kn, alpha, beta = prologue(q, k, a, b, qk_l2norm, gate_logits, alpha_scale)
    o, S = prefill_sequential(qn, kn, v, alpha, beta, S0=S0, per_key=per_key, order=order)
    if z is not None:
        o = output_gate(o, z)
    return o, S


def decode(q, k, v, a, b, S, z=None, per_key=False, order="delta_first", qk_l2norm=True,
           gate_logits=True, alpha_scale=1.0):
    """One decode token per unit with the same prologue and epilogue.  Returns (o, S_new)."""
    qn, kn, alpha, beta = prologue(q, k, a, b, qk_l2norm, gate_logits, alpha_scale)
    o, S_new = decode_step(qn, kn, v, alpha, beta, S, per_key=per_key, order=order)
    if z is not None:
        o = output_gate(o, z)
    return o, S_new
