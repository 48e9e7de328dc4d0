"""fp64 oracle of the looped prefill over packed sequences of different lengths (test
infrastructure only).

The product path never imports this module.  "LT2 transformer looped a tempo lineare", section
"Sostituire il motore", displayed equation: the recurrence runs over the tokens of one sequence
from its own initial state.  A packed ("varlen") batch holds B sequences one after the other
along a token axis of length Ntot, sequence b owning tokens cu[b] .. cu[b+1]-1; every (loop,
sequence, head) is its own recurrence, so the oracle is the definition applied to each
sequence's slice in turn:

    q, k [T, H, Ntot, d_k], v [T, H, Ntot, d_v], alpha [T, H, Ntot] (or [..., d_k] per key),
    beta [T, H, Ntot], S0 [T, B, H, d_k, d_v] or None  ->  o [T, H, Ntot, d_v], S [T, B, H, d_k, d_v]

The sequential oracle (``oracle.prefill_sequential``) or, with raw inputs, the fused one
(``oracle.fused.prefill``) does each slice; nothing here computes more than the slicing.
"""
import numpy as np

from . import prefill_sequential
from . import fused as _fused


def _slice(x, c0, c1):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64)[:, :, c0:c1])


def prefill(q, k, v, alpha, beta, cu_seqlens, S0=None, per_key=False, order="delta_first",
            raw=None):
    """Per-sequence recurrence over a packed batch.  ``raw`` = dict(z=..., qk_l2norm=...,
    gate_logits=..., alpha_scale=...) runs the fused prologue and output gate instead (alpha and
    beta then hold the logits a and b)."""
    q = np.asarray(q, dtype=np.float64)
    T, H, N, dk = q.shape
    dv = np.shape(v)[-1]
    cu = [int(c) for c in np.asarray(cu_seqlens).ravel()]
    B = len(cu) - 1
    o = np.zeros((T, H, N, dv))
    S = np.zeros((T, B, H, dk, dv))
    for b in range(B):
        c0, c1 = cu[b], cu[b + 1]
        s0 = None if S0 is None else np.ascontiguousarray(np.asarray(S0, dtype=np.float64)[:, b])
        if c1 == c0:
            S[:, b] = 0.0 if s0 is None else s0
            continue
        args = [_slice(x, c0, c1) for x in (q, k, v, alpha, beta)]
        if raw is None:
            ob, Sb = prefill_sequential(*args, S0=s0, per_key=per_key, order=order)
        else:
            ob, Sb = _fused.prefill(*args, z=_slice(raw.get("z"), c0, c1), S0=s0, per_key=per_key,
                                    order=order, qk_l2norm=raw.get("qk_l2norm", True),
                                    gate_logits=raw.get("gate_logits", True),
                                    alpha_scale=raw.get("alpha_scale", 1.0))
        o[:, :, c0:c1] = ob
        S[:, b] = Sb
    return o, S
