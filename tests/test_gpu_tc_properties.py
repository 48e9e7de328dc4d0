"""The recurrence's own properties on the tensor-core prefills (d = 128, bf16 inputs), for
scalar gating and for per-key gating in both orders of the factors.

"LT2 transformer looped a tempo lineare", section "Sostituire il motore", displayed equation:
S_t = Diag(alpha_t)(I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, read out as o_t = S_t^T q_t.

- beta = 0: the state only decays, S_t = Gamma_t S_0 with Gamma_t = Diag(prod_{s<=t} alpha_s),
  and o_t = S_0^T Gamma_t q_t.
- mutually orthogonal unit keys and S_0 = 0: no write is ever projected away, so the readout is
  decayed linear attention, o_t = sum_{s<=t} beta_s (decay of key i_s from s+1 to t) (q_t . k_s) v_s.
- alpha = 0 (a reset) and alpha < 0 in the scalar kernel, against the fp64 oracle.
- a state growing past the fp16 range of the tensor-core operands: the call either matches the
  oracle or reports LT2_ERR_RANGE, never silent infinities.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill, to_np

pytestmark = pytest.mark.gpu

TC = lt2.LT2_ALGO_TENSOR_CORE
GATES = [("scalar", "delta_first"), ("per_key", "delta_first"), ("per_key", "decay_first")]


def _inputs(gate, T=2, B=1, H=3, L=200, seed=0, s0="normal"):
    name = "kda_prefill" if gate == "per_key" else "gdn_prefill"
    w = inputs.workload(name, T=T, B=B, H=H, L=L, s0=s0)
    return inputs.make_inputs(w, seed=seed, device="cuda")


def _run(x, gate, order, algo=TC, check_status=True):
    o, S = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x.get("S0"),
                       per_key=gate == "per_key", algo=algo, out="f32", order=order)
    torch.cuda.synchronize()
    st = lt2.lt2_gdr_last_device_error()
    if check_status:
        assert st == lt2.LT2_OK, lt2.lt2_status_string(st)
    return o, S, st


def _cumdecay(alpha, per_key):
    """Gamma_t (inclusive running product of alpha over tokens), fp64, [..., L, d_k]."""
    a = to_np(alpha)
    if not per_key:
        a = a[..., None]
    return np.cumprod(a, axis=-2)


@pytest.mark.parametrize("gate,order", GATES)
def test_beta_zero_only_decays(gate, order):
    x = _inputs(gate, L=200, seed=3)
    x["beta"].zero_()
    o, S, _ = _run(x, gate, order)
    per_key = gate == "per_key"
    G = _cumdecay(x["alpha"], per_key)                 # [T,B,H,L,dk or 1]
    S0, q = to_np(x["S0"]), to_np(x["q"])
    # o_t = S0^T (Gamma_t q_t);  S_L = Gamma_L S0
    o_ref = np.einsum("tbhkv,tbhlk->tbhlv", S0, G * q)
    S_ref = G[..., -1, :, None] * S0
    check("o (beta = 0)", o, o_ref, TOL["bf16"])
    check("S_T (beta = 0)", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate,order", GATES)
def test_orthogonal_keys_give_decayed_linear_attention(gate, order):
    T, B, H, L, d = 2, 1, 2, 128, 128
    x = _inputs(gate, T=T, B=B, H=H, L=L, seed=5, s0="zeros")
    # signed, permuted standard-basis keys: mutually orthogonal, unit norm, exact in bf16
    rng = np.random.default_rng(11)
    idx = np.stack([rng.permutation(d)[:L] for _ in range(T * B * H)]).reshape(T, B, H, L)
    sgn = rng.choice([-1.0, 1.0], size=(T, B, H, L))
    k = np.zeros((T, B, H, L, d))
    np.put_along_axis(k, idx[..., None], sgn[..., None], axis=-1)
    x["k"] = torch.tensor(k, dtype=torch.bfloat16, device="cuda")
    o, S, _ = _run(x, gate, order)
    per_key = gate == "per_key"
    G = _cumdecay(x["alpha"], per_key)                 # inclusive products
    q, v, beta = to_np(x["q"]), to_np(x["v"]), to_np(x["beta"])
    o_ref = np.zeros((T, B, H, L, d))
    S_ref = np.zeros((T, B, H, d, d))
    for u in np.ndindex(T, B, H):
        g = G[u]                                       # [L, dk or 1]
        col = (lambda t, i: g[t, i]) if per_key else (lambda t, i: g[t, 0])
        for t in range(L):
            acc = np.zeros(d)
            for s in range(t + 1):
                i = idx[u][s]
                acc += beta[u][s] * (col(t, i) / col(s, i)) * sgn[u][s] * q[u][t, i] * v[u][s]
            o_ref[u][t] = acc
        for s in range(L):
            i = idx[u][s]
            S_ref[u][i] += beta[u][s] * (col(L - 1, i) / col(s, i)) * sgn[u][s] * v[u][s]
    check("o (orthogonal keys)", o, o_ref, TOL["bf16"])
    check("S_T (orthogonal keys)", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("L", [64, 200])
def test_scalar_resets_and_negative_alpha(L):
    x = _inputs("scalar", H=4, L=L, seed=7)
    a = x["alpha"]
    a[..., 5] = 0.0                                    # resets
    a[..., 37] = 0.0
    a[0, 0, 1, 10:20] = -a[0, 0, 1, 10:20]             # a run of negative decays
    a[1, 0, 2, 60] = -0.5
    a[1, 0, 3, :] = 0.0                                # every token a reset
    o, S, _ = _run(x, "scalar", "delta_first")
    o_ref, S_ref = oracle_prefill(x, per_key=False)
    check("o (resets, alpha < 0)", o, o_ref, TOL["bf16"])
    check("S_T (resets, alpha < 0)", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate,order", GATES)
def test_growth_past_fp16_is_reported(gate, order):
    # alpha = 1.06 on every token: the state grows ~1.06^t, past the fp16 range within 512
    # tokens.  The exact result is finite; the tensor-core path must flag it or match it.
    x = _inputs(gate, T=1, H=2, L=512, seed=9, s0="zeros")
    x["alpha"].fill_(1.06)
    o, S, st = _run(x, gate, order, check_status=False)
    o_ref, S_ref = oracle_prefill(x, per_key=gate == "per_key", order=order)
    assert np.isfinite(o_ref).all() and np.abs(S_ref).max() > 7e4
    if st == lt2.LT2_OK:
        check("o (growth)", o, o_ref, TOL["bf16"])
        check("S_T (growth)", S, S_ref, TOL["bf16"])
    else:
        assert st == lt2.LT2_ERR_RANGE, lt2.lt2_status_string(st)
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK       # read once, then cleared
    # the fp32 CUDA-core path computes the same call
    o32, S32, _ = _run(x, gate, order, algo=lt2.LT2_ALGO_CUDA_CORE)
    check("o (growth, cuda core)", o32, o_ref, 1e-3)
    check("S_T (growth, cuda core)", S32, S_ref, 1e-3)


def test_range_flag_leaves_the_next_call_clean():
    x = _inputs("scalar", T=1, H=2, L=512, seed=9, s0="zeros")
    x["alpha"].fill_(1.06)
    _run(x, "scalar", "delta_first", check_status=False)
    y = _inputs("scalar", T=1, H=2, L=130, seed=1)
    o, S, st = _run(y, "scalar", "delta_first")
    o_ref, S_ref = oracle_prefill(y, per_key=False)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])
