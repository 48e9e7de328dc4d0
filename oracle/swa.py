"""fp64 oracle of the looped sliding-window attention mixer (test infrastructure only).

The product path never imports this module.  "LT2 transformer looped a tempo lineare",
section "Sostituire il motore": the second family of sub-quadratic mixers is sparse attention,
in which every token looks only at a window of the w most recent positions instead of the whole
history; section "Il giro trasforma il calcolo in contesto": a window of width w, repeated T
times, reaches back O(T w) tokens, because at every loop each position absorbs neighbours that
had already absorbed their own.

Readings (the pages give no formula): the window of token t is positions t - w + 1 .. t (the
token itself included, w positions at most, fewer at the start of the sequence); the weights
are the softmax over that window of scale * q_t . k_s, with scale = 1 / sqrt(d_k) unless one is
given; o_t = sum_s weight_s v_s.  As for the linear mixer, every (loop, batch, head) is
independent in the isolated mixer: each loop comes with its own q, k, v.

Entry points take numpy arrays [..., L, d] (any leading dims, each an independent unit) and
return fp64:
    prefill(q, k, v, window, scale=None)        the definition, one query at a time
    prefill_dense(q, k, v, window, scale=None)  the same through a full L x L masked score matrix
"""
import math

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def default_scale(dk):
    return 1.0 / math.sqrt(dk)


def prefill(q, k, v, window, scale=None):
    """o_t = softmax_{s in [t-w+1, t]}(scale q_t . k_s) v_s for every t, per unit."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    L, dk = q.shape[-2:]
    scale = default_scale(dk) if scale is None else float(scale)
    lead = q.shape[:-2]
    qf, kf, vf = q.reshape(-1, L, dk), k.reshape(-1, L, dk), v.reshape(-1, L, v.shape[-1])
    o = np.zeros(vf.shape)
    w = int(window)
    for u in range(qf.shape[0]):
        for t in range(L):
            s0 = max(0, t - w + 1)
            sc = scale * (kf[u, s0:t + 1] @ qf[u, t])
            p = np.exp(sc - sc.max())
            o[u, t] = (p / p.sum()) @ vf[u, s0:t + 1]
    return o.reshape(lead + (L, v.shape[-1]))


def prefill_dense(q, k, v, window, scale=None):
    """The same as one masked L x L matrix per unit (brute force, for cross-checks)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    L, dk = q.shape[-2:]
    scale = default_scale(dk) if scale is None else float(scale)
    t = np.arange(L)[:, None]
    s = np.arange(L)[None, :]
    allowed = (s <= t) & (s > t - int(window))
    sc = scale * np.einsum("...td,...sd->...ts", q, k)
    sc = np.where(allowed, sc, -np.inf)
    sc = sc - sc.max(axis=-1, keepdims=True)
    p = np.exp(sc)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("...ts,...sd->...td", p, v)
