"""fp64 CPU oracle for the looped gated delta rule (LT2 linear mixer).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``.  The product path never imports it, and it imports nothing
from the product package.

The recurrence ("LT2 transformer looped a tempo lineare", section "Sostituire il motore",
displayed equation), per independent (loop, batch, head) unit:

    S_t = Diag(alpha_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t

Entry points take numpy arrays shaped ``[..., L, d]`` (any leading dims, flattened into
independent head-units), up-cast everything to fp64 and return fp64 results:

    prefill_sequential   the equation token by token (primary oracle)
    prefill_dense        A_t built as a dense matrix (brute force cross-check)
    prefill_chunked      chunk-parallel UT/WY rewriting (u-form or e-form)
    decode_step          one token, state updated and returned

``oracle.twin`` holds a second, pure numpy implementation for tiny cases.

Order of the per-key factors.  ``order="delta_first"`` (the default) is the equation as printed,
A_t = Diag(alpha_t)(I - beta_t k_t k_t^T).  ``order="decay_first"`` takes
A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), the order a right-multiplying convention for the
state would give; the page's equation fixes the first, the second is the other reading of the
same symbols.  For scalar gating both are the same matrix.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIBS = {}


def _lib(path=None):
    """The compiled oracle at ``path`` (default: oracle/_build/libgdr_oracle.so, built on
    first use).  Tests that plant mistakes pass the path of a deliberately broken copy."""
    key = path or _build.OUT
    if key not in _LIBS:
        if path is None and _build.needs_build():
            _build.build()
        lib = ctypes.CDLL(key)
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        common = [i64, i64, i64, i64, ctypes.c_int]
        tail = [dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.gdr_ref_sequential.argtypes = common + tail
        lib.gdr_ref_dense.argtypes = common + tail
        lib.gdr_ref_chunked.argtypes = common + [i64, ctypes.c_int] + tail
        for f in (lib.gdr_ref_sequential, lib.gdr_ref_dense, lib.gdr_ref_chunked):
            f.restype = ctypes.c_int
        lib.gdr_ref_threads.argtypes = [ctypes.c_int]
        lib.gdr_ref_threads.restype = ctypes.c_int
        _LIBS[key] = lib
    return _LIBS[key]


def threads(nthreads=0):
    """Number of OpenMP threads a call with ``nthreads`` (0 = default) will use."""
    return _lib().gdr_ref_threads(int(nthreads))


def _f64(x):
    a = np.asarray(x, dtype=np.float64)
    return a if a.flags.c_contiguous else a.copy(order="C")


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _gate_code(per_key, order):
    """Gate code of the C oracle: 0 scalar, 1 per-key delta first, 2 per-key decay first."""
    if order not in ("delta_first", "decay_first"):
        raise ValueError(f"order must be 'delta_first' or 'decay_first', got {order!r}")
    if not per_key:
        return 0
    return 2 if order == "decay_first" else 1


def _prep(q, k, v, alpha, beta, S0, per_key):
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    if q.shape != k.shape or q.ndim < 2:
        raise ValueError("q and k must share a [..., L, d_k] shape")
    lead = q.shape[:-2]
    L, dk = q.shape[-2:]
    if v.shape[:-1] != q.shape[:-1]:
        raise ValueError("v must be [..., L, d_v] with q's leading shape")
    dv = v.shape[-1]
    want_alpha = q.shape if per_key else q.shape[:-1]
    if alpha.shape != want_alpha:
        raise ValueError(f"alpha must be {want_alpha}, got {alpha.shape}")
    if beta.shape != q.shape[:-1]:
        raise ValueError(f"beta must be {q.shape[:-1]}, got {beta.shape}")
    U = int(np.prod(lead)) if lead else 1
    if S0 is not None:
        S0 = _f64(S0)
        if S0.shape != lead + (dk, dv):
            raise ValueError(f"S0 must be {lead + (dk, dv)}, got {S0.shape}")
    o = np.zeros(lead + (L, dv), dtype=np.float64)
    S = np.zeros(lead + (dk, dv), dtype=np.float64)
    return q, k, v, alpha, beta, S0, o, S, U, L, dk, dv


def prefill_sequential(q, k, v, alpha, beta, S0=None, per_key=False, nthreads=0, lib=None,
                       order="delta_first"):
    """Token-by-token recurrence. Returns (o [..., L, d_v], S_L [..., d_k, d_v]) in fp64."""
    g = _gate_code(per_key, order)
    q, k, v, alpha, beta, S0, o, S, U, L, dk, dv = _prep(q, k, v, alpha, beta, S0, per_key)
    rc = _lib(lib).gdr_ref_sequential(U, L, dk, dv, g, _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S),
                                   int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdr_ref_sequential failed ({rc})")
    return o, S


def prefill_dense(q, k, v, alpha, beta, S0=None, per_key=False, nthreads=0, order="delta_first"):
    """Same recurrence with A_t materialised as a d_k x d_k matrix (brute force)."""
    g = _gate_code(per_key, order)
    q, k, v, alpha, beta, S0, o, S, U, L, dk, dv = _prep(q, k, v, alpha, beta, S0, per_key)
    rc = _lib().gdr_ref_dense(U, L, dk, dv, g, _ptr(q), _ptr(k), _ptr(v),
                              _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S),
                              int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdr_ref_dense failed ({rc})")
    return o, S


def prefill_chunked(q, k, v, alpha, beta, S0=None, per_key=False, chunk=64, form="e",
                    nthreads=0, order="delta_first"):
    """Chunk-parallel rewriting; ``form`` is "u" (scalar gating only), "wy" (the u-form with
    T = (I + A)^{-1} written out, one product with S0 per chunk; scalar gating only) or "e"
    (either gating)."""
    g = _gate_code(per_key, order)
    q, k, v, alpha, beta, S0, o, S, U, L, dk, dv = _prep(q, k, v, alpha, beta, S0, per_key)
    f = {"u": 0, "e": 1, "wy": 2}[form]
    rc = _lib().gdr_ref_chunked(U, L, dk, dv, g, int(chunk), f, _ptr(q), _ptr(k),
                                _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S),
                                int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdr_ref_chunked failed ({rc})")
    return o, S


def decode_step(q, k, v, alpha, beta, S, per_key=False, nthreads=0, lib=None, order="delta_first"):
    """One token per unit. q, k: [..., d_k]; v: [..., d_v]; alpha: [...] or [..., d_k];
    beta: [...]; S: [..., d_k, d_v].  Returns (o [..., d_v], S_new)."""
    q = _f64(q)[..., None, :]
    k = _f64(k)[..., None, :]
    v = _f64(v)[..., None, :]
    alpha = _f64(alpha)
    alpha = alpha[..., None, :] if per_key else alpha[..., None]
    beta = _f64(beta)[..., None]
    o, S_new = prefill_sequential(q, k, v, alpha, beta, S0=S, per_key=per_key,
                                  nthreads=nthreads, lib=lib, order=order)
    return o[..., 0, :], S_new


def rel_max_err(x, ref):
    """max |x - ref| / rms(ref) over the whole tensor (the parity metric)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    if rms == 0.0:
        return err
    return err / rms
