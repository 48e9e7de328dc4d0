"""The fused prologue and output gate (lt2_gdr_prefill_fused / lt2_gdr_decode_fused) on every
path, against the fp64 oracle of oracle/fused.py on the same raw inputs.

Raw inputs: q, k ~ N(0,1) (norm ~ sqrt(d), normalised inside), gate logits a, b ~ N(0,1)
(alpha = exp(-softplus(a) c), beta = sigmoid(b), c = 0.1 as the workloads), output gate logits
z ~ N(0,1) (o <- sigmoid(z) o: "LT2 transformer looped a tempo lineare", section "Dove il
quadro si incrina").
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from oracle import fused as ofused
from tests.gpu_util import TOL, check, to_np

pytestmark = pytest.mark.gpu

C = 0.1
TC, CC = lt2.LT2_ALGO_TENSOR_CORE, lt2.LT2_ALGO_CUDA_CORE
PATHS = [("scalar", "delta_first", TC), ("per_key", "delta_first", TC), ("per_key", "decay_first", TC),
         ("scalar", "delta_first", CC), ("per_key", "delta_first", CC), ("per_key", "decay_first", CC)]


def _raw(gate, L, seed, T=2, H=2, dtype="bf16", d=128):
    w = inputs.workload("kda_prefill" if gate == "per_key" else "gdn_prefill", T=T, B=1, H=H, L=L,
                        s0="normal", dtype=dtype, d=d)
    return inputs.make_raw_inputs(w, seed=seed, device="cuda")


def _oracle(x, gate, order, norm=True, logits=True, gated=True):
    return ofused.prefill(to_np(x["q"]), to_np(x["k"]), to_np(x["v"]), to_np(x["a"]), to_np(x["b"]),
                          z=to_np(x["z"]) if gated else None, S0=to_np(x["S0"]), per_key=gate == "per_key",
                          order=order, qk_l2norm=norm, gate_logits=logits, alpha_scale=C)


def _run(x, gate, order, algo, norm=True, logits=True, gated=True, out="f32"):
    o, S = lt2.prefill(x["q"], x["k"], x["v"], x["a"], x["b"], S0=x["S0"], per_key=gate == "per_key",
                       algo=algo, out=out, order=order, qk_l2norm=norm, gate_logits=logits, alpha_scale=C,
                       z=x["z"] if gated else None)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    return o, S


@pytest.mark.parametrize("gate,order,algo", PATHS)
@pytest.mark.parametrize("L", [1, 65, 200])
def test_fused_prefill_matches_oracle(gate, order, algo, L):
    x = _raw(gate, L, seed=L + 3)
    o, S = _run(x, gate, order, algo)
    o_ref, S_ref = _oracle(x, gate, order)
    check("o (fused)", o, o_ref, TOL["bf16"])
    check("S_T (fused)", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate,order,algo", [p for p in PATHS if p[2] == TC])
@pytest.mark.parametrize("norm,logits,gated", [(True, False, False), (False, True, False), (False, False, True)])
def test_each_fused_step_alone(gate, order, algo, norm, logits, gated):
    x = _raw(gate, 130, seed=5)
    if not norm:                       # the recurrence needs unit keys when they are not normalised inside
        x["q"] = (x["q"].float() / x["q"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        x["k"] = (x["k"].float() / x["k"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    if not logits:
        x["a"] = torch.exp(-torch.nn.functional.softplus(x["a"]) * C)
        x["b"] = torch.sigmoid(x["b"])
    o, S = _run(x, gate, order, algo, norm, logits, gated)
    o_ref, S_ref = _oracle(x, gate, order, norm, logits, gated)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate,order", [("scalar", "delta_first"), ("per_key", "delta_first"), ("per_key", "decay_first")])
def test_fused_fp32_cuda_core_is_exact(gate, order):
    # fp32 inputs on the CUDA-core path: the 1e-4 bar, with the accurate exp / log1p / sqrt
    x = _raw(gate, 77, seed=9, dtype="f32", d=32)
    o, S = _run(x, gate, order, lt2.LT2_ALGO_AUTO)
    o_ref, S_ref = _oracle(x, gate, order)
    check("o (fp32)", o, o_ref, TOL["f32"])
    check("S_T (fp32)", S, S_ref, TOL["f32"])


@pytest.mark.parametrize("gate,order,algo", [p for p in PATHS if p[2] == TC])
def test_fused_bf16_output_is_rounded_fp32_output(gate, order, algo):
    x = _raw(gate, 150, seed=13)
    o32, S32 = _run(x, gate, order, algo, out="f32")
    o16, S16 = _run(x, gate, order, algo, out="bf16")
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S32)


@pytest.mark.parametrize("gate,order", [("scalar", "delta_first"), ("per_key", "delta_first"), ("per_key", "decay_first")])
@pytest.mark.parametrize("dtype,tol", [("bf16", TOL["bf16"]), ("f32", TOL["f32"])])
def test_fused_decode_matches_oracle(gate, order, dtype, tol):
    x = _raw(gate, 1, seed=21, T=2, H=3, dtype=dtype)
    one = {n: (t[..., 0, :] if n in ("q", "k", "v", "z") or (n == "a" and gate == "per_key") else t[..., 0])
           for n, t in x.items() if n != "S0"}
    S = x["S0"].clone()
    o = lt2.decode(one["q"], one["k"], one["v"], one["a"], one["b"], S, per_key=gate == "per_key",
                   out="f32", order=order, qk_l2norm=True, gate_logits=True, alpha_scale=C, z=one["z"])
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    o_ref, S_ref = ofused.decode(to_np(one["q"]), to_np(one["k"]), to_np(one["v"]), to_np(one["a"]),
                                 to_np(one["b"]), to_np(x["S0"]), z=to_np(one["z"]), per_key=gate == "per_key",
                                 order=order, alpha_scale=C)
    check("o (fused decode)", o, o_ref, tol)
    check("S (fused decode)", S, S_ref, tol)


def test_fused_full_size_gdn_prefill_sampled_units():
    # the gdn_prefill shape (T4 B4 H16 L8192) with raw inputs, every loop launch in one call;
    # one unit of every loop checked against the oracle
    w = inputs.workload("gdn_prefill")
    x = inputs.make_raw_inputs(w, seed=0, device="cuda")
    o, S = lt2.prefill(x["q"], x["k"], x["v"], x["a"], x["b"], per_key=False, out="f32", qk_l2norm=True,
                       gate_logits=True, alpha_scale=C, z=x["z"])
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    rng = np.random.default_rng(2)
    units = sorted({(t, int(rng.integers(w.B)), int(rng.integers(w.H))) for t in range(w.T)} | {(0, 0, 0)})
    sel = lambda t: torch.stack([t[u] for u in units])
    o_ref, S_ref = ofused.prefill(to_np(sel(x["q"])), to_np(sel(x["k"])), to_np(sel(x["v"])), to_np(sel(x["a"])),
                                  to_np(sel(x["b"])), z=to_np(sel(x["z"])), alpha_scale=C)
    check("o (sampled units)", sel(o), o_ref, TOL["bf16"])
    check("S_T (sampled units)", sel(S), S_ref, TOL["bf16"])
