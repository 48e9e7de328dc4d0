"""Pure numpy twin of the oracle, for tiny cases (test infrastructure only).

Written independently of ``gdr_oracle.c``: it forms the transition matrix
A_t = Diag(alpha_t) (I - beta_t k_t k_t^T) with numpy and applies
S_t = A_t S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t
("LT2 transformer looped a tempo lineare", section "Sostituire il motore", displayed
equation), one head-unit at a time with Python loops.
"""
import numpy as np


def prefill(q, k, v, alpha, beta, S0=None, per_key=False, order="delta_first"):
    """``order="decay_first"`` takes A_t = (I - beta_t k_t k_t^T) Diag(alpha_t) instead."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    lead = q.shape[:-2]
    L, dk = q.shape[-2:]
    dv = v.shape[-1]
    U = int(np.prod(lead)) if lead else 1
    qf = q.reshape(U, L, dk)
    kf = k.reshape(U, L, dk)
    vf = v.reshape(U, L, dv)
    af = alpha.reshape(U, L, dk) if per_key else alpha.reshape(U, L)
    bf = beta.reshape(U, L)
    S0f = None if S0 is None else np.asarray(S0, dtype=np.float64).reshape(U, dk, dv)
    o = np.zeros((U, L, dv))
    S_out = np.zeros((U, dk, dv))
    eye = np.eye(dk)
    for u in range(U):
        S = np.zeros((dk, dv)) if S0f is None else S0f[u].copy()
        for t in range(L):
            kt = kf[u, t]
            diag = af[u, t] if per_key else np.full(dk, af[u, t])
            delta = eye - bf[u, t] * np.outer(kt, kt)
            A = delta @ np.diag(diag) if order == "decay_first" else np.diag(diag) @ delta
            S = A @ S + bf[u, t] * np.outer(kt, vf[u, t])
            o[u, t] = S.T @ qf[u, t]
        S_out[u] = S
    return o.reshape(lead + (L, dv)), S_out.reshape(lead + (dk, dv))
