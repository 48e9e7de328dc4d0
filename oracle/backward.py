"""fp64 oracle of the backward pass of the looped gated delta rule (test infrastructure only).

The product path never imports this module.  The forward recurrence is the displayed equation of
"LT2 transformer looped a tempo lineare", section "Sostituire il motore", per (loop, batch, head)
unit, with the readout after the update:

    printed order (delta, then decay):  e_t = S_{t-1}^T k_t,
        P_t = S_{t-1} - beta_t k_t e_t^T,     S_t = Diag(alpha_t) P_t + beta_t k_t v_t^T
    decay-first order:                  R_t = Diag(alpha_t) S_{t-1},  e_t = R_t^T k_t,
        S_t = R_t - beta_t k_t e_t^T + beta_t k_t v_t^T
    o_t = S_t^T q_t

(alpha_t a scalar or a d_k vector).  The pages train looped models but give no training kernel,
so the backward pass is the plain reverse-mode derivative of that recurrence: for a loss with
upstream gradients dO_t = dLoss/do_t and dS_L = dLoss/dS_L, a sweep from t = L down to 1 carries
G = dLoss/dS_t and produces dq_t, dk_t, dv_t, dalpha_t, dbeta_t, and finally dS_0 = G.  Each step
below is the derivative of one line of the forward step (written out, one token at a time); the
test suite checks every gradient against central finite differences of the forward oracle.

    G   += q_t dO_t^T                           (o_t = S_t^T q_t)
    dq_t = S_t dO_t
    printed order, with dP = Diag(alpha_t) G:
        dv_t      = beta_t G^T k_t
        dbeta_t   = k_t^T G v_t - (k_t^T dP) . e_t
        dk_t      = beta_t G v_t - beta_t (S_{t-1} (dP^T k_t) + dP e_t)
        dalpha_t  = rowsum(G * P_t)  (scalar alpha: the sum of all entries)
        G        <- dP - beta_t k_t (k_t^T dP)
    decay-first order, with kG = G^T k_t and dR = G - beta_t k_t kG^T:
        dv_t      = beta_t kG
        dbeta_t   = kG . (v_t - e_t)
        dk_t      = beta_t G (v_t - e_t) - beta_t R_t kG
        dalpha_t  = rowsum(dR * S_{t-1})  (scalar alpha: the sum of all entries)
        G        <- Diag(alpha_t) dR

Entry point (numpy arrays, any leading dims, each an independent unit):
    backward(q, k, v, alpha, beta, dO, S0=None, dS_L=None, per_key=False, order="delta_first")
        -> dict(dq, dk, dv, dalpha, dbeta, dS0) in fp64
"""
import numpy as np


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _unit_backward(q, k, v, al, be, dO, S0, dSL, per_key, decay_first):
    L, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((L + 1, dk, dv))
    S[0] = 0.0 if S0 is None else S0
    for t in range(L):                                   # forward, keeping every state
        a = al[t] if per_key else np.full(dk, al[t])
        if decay_first:
            R = a[:, None] * S[t]
            e = R.T @ k[t]
            S[t + 1] = R + be[t] * np.outer(k[t], v[t] - e)
        else:
            e = S[t].T @ k[t]
            S[t + 1] = a[:, None] * (S[t] - be[t] * np.outer(k[t], e)) + be[t] * np.outer(k[t], v[t])
    G = np.zeros((dk, dv)) if dSL is None else np.array(dSL, dtype=np.float64)
    dq = np.zeros((L, dk))
    dkk = np.zeros((L, dk))
    dvv = np.zeros((L, dv))
    dal = np.zeros((L, dk)) if per_key else np.zeros(L)
    dbe = np.zeros(L)
    for t in range(L - 1, -1, -1):
        a = al[t] if per_key else np.full(dk, al[t])
        kt, vt, b = k[t], v[t], be[t]
        G = G + np.outer(q[t], dO[t])
        dq[t] = S[t + 1] @ dO[t]
        if decay_first:
            R = a[:, None] * S[t]
            e = R.T @ kt
            kG = G.T @ kt
            dR = G - b * np.outer(kt, kG)
            dvv[t] = b * kG
            dbe[t] = kG @ (vt - e)
            dkk[t] = b * (G @ (vt - e)) - b * (R @ kG)
            da = np.sum(dR * S[t], axis=1)
            G = a[:, None] * dR
        else:
            e = S[t].T @ kt
            P = S[t] - b * np.outer(kt, e)
            dP = a[:, None] * G
            kdP = dP.T @ kt
            dvv[t] = b * (G.T @ kt)
            dbe[t] = kt @ G @ vt - kdP @ e
            dkk[t] = b * (G @ vt) - b * (S[t] @ kdP + dP @ e)
            da = np.sum(G * P, axis=1)
            G = dP - b * np.outer(kt, kdP)
        dal[t] = da if per_key else np.sum(da)
    return dq, dkk, dvv, dal, dbe, G


def backward(q, k, v, alpha, beta, dO, S0=None, dS_L=None, per_key=False, order="delta_first"):
    """Gradients of sum(dO * o) + sum(dS_L * S_L) w.r.t. q, k, v, alpha, beta and S0."""
    if order not in ("delta_first", "decay_first"):
        raise ValueError(order)
    q, k, v, alpha, beta, dO, S0, dS_L = (_f64(x) for x in (q, k, v, alpha, beta, dO, S0, dS_L))
    L, dk = q.shape[-2:]
    dv = v.shape[-1]
    lead = q.shape[:-2]
    U = int(np.prod(lead)) if lead else 1
    f = lambda x, *tail: None if x is None else x.reshape((U,) + tail)
    qf, kf, vf, dOf = f(q, L, dk), f(k, L, dk), f(v, L, dv), f(dO, L, dv)
    af = f(alpha, L, dk) if per_key else f(alpha, L)
    bf = f(beta, L)
    S0f, dSf = f(S0, dk, dv), f(dS_L, dk, dv)
    out = {n: [] for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")}
    for u in range(U):
        r = _unit_backward(qf[u], kf[u], vf[u], af[u], bf[u], dOf[u], None if S0f is None else S0f[u],
                           None if dSf is None else dSf[u], per_key, order == "decay_first")
        for n, x in zip(out, r):
            out[n].append(x)
    shapes = {"dq": (L, dk), "dk": (L, dk), "dv": (L, dv), "dalpha": (L, dk) if per_key else (L,),
              "dbeta": (L,), "dS0": (dk, dv)}
    return {n: np.stack(x).reshape(lead + shapes[n]) for n, x in out.items()}
