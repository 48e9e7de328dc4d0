"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on the same seeded
inputs, element by element, with the tolerance max|gpu - ref| / rms(ref) <= 1e-4 for fp32
inputs and <= 2e-2 for bf16 inputs with fp32 state (checked on o and the final state
separately).  o is compared in its fp32 form; a bf16 o must equal that fp32 o rounded to
nearest-even, bit for bit."""
import dataclasses

import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
import oracle
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill, run_prefill, to_device, to_np

pytestmark = pytest.mark.gpu

ALGOS = [lt2.LT2_ALGO_AUTO, lt2.LT2_ALGO_CUDA_CORE]


def _case(name, seed=0, **over):
    w = inputs.workload(name, **over)
    x = inputs.make_inputs(w, seed=seed, device="cpu")
    return w, to_device(x)


def test_tiny_fp32_workload():
    # The tiny oracle case exactly: T=2 B=1 H=2 L=64 d=32, fp32, S0 = 0.
    w, x = _case("tiny_fp32")
    o, S = run_prefill(x, per_key=False)
    o_ref, S_ref = oracle_prefill(x, False)
    check("o", o, o_ref, TOL["f32"])
    check("S_T", S, S_ref, TOL["f32"])


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("per_key", [False, True])
@pytest.mark.parametrize("L", [1, 63, 200])
def test_bf16_d128_small(algo, per_key, L):
    name = "kda_prefill" if per_key else "gdn_prefill"
    w, x = _case(name, seed=L, T=2, B=1, H=2, L=L, s0="normal")
    o, S = run_prefill(x, per_key=per_key, algo=algo)
    o_ref, S_ref = oracle_prefill(x, per_key)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(8, 8), (64, 32), (32, 128), (128, 64)])
@pytest.mark.parametrize("per_key", [False, True])
def test_fp32_shapes(dk, dv, per_key):
    w = dataclasses.replace(inputs.workload("tiny_fp32"), d=dk, L=77, s0="normal",
                            gate="per_key" if per_key else "scalar")
    x = inputs.make_inputs(w, seed=dk + dv)
    # v with a different width than q/k
    g = torch.Generator().manual_seed(5)
    x["v"] = torch.randn(x["q"].shape[:-1] + (dv,), generator=g)
    x["S0"] = torch.randn(x["q"].shape[:3] + (dk, dv), generator=g)
    x = to_device(x)
    o, S = run_prefill(x, per_key=per_key)
    o_ref, S_ref = oracle_prefill(x, per_key)
    check("o", o, o_ref, TOL["f32"])
    check("S_T", S, S_ref, TOL["f32"])


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("per_key", [False, True])
def test_bf16_output_is_rounded_fp32_output(algo, per_key):
    name = "kda_prefill" if per_key else "gdn_prefill"
    w, x = _case(name, seed=21, T=2, B=1, H=2, L=130)
    o32, S32 = run_prefill(x, per_key=per_key, algo=algo, out="f32")
    o16, S16 = run_prefill(x, per_key=per_key, algo=algo, out="bf16")
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S16, S32)


def test_empty_sequence_copies_state():
    w, x = _case("gdn_prefill", T=1, B=1, H=2, L=0, s0="normal")
    o, S = run_prefill(x, per_key=False)
    assert o.numel() == 0
    assert torch.equal(S, x["S0"])


def test_in_place_resume_equals_full_prefill():
    # S0 == S_out (documented in-place resume) and segment resume: prefill(L1) then
    # prefill(L2, S0 = S_L1) reproduces prefill(L1 + L2).
    w, x = _case("gdn_prefill", seed=3, T=2, B=1, H=2, L=150)
    o_full, S_full = run_prefill(x, per_key=False)
    cut = 70
    xa = {k: (v[:, :, :, :cut] if k in ("q", "k", "v", "alpha", "beta") else v) for k, v in x.items()}
    xb = {k: (v[:, :, :, cut:].contiguous() if k in ("q", "k", "v", "alpha", "beta") else v)
          for k, v in x.items()}
    xa = {k: (v.contiguous() if isinstance(v, torch.Tensor) else v) for k, v in xa.items()}
    oa, Sa = run_prefill(xa, per_key=False)
    ob, _ = lt2.prefill(xb["q"], xb["k"], xb["v"], xb["alpha"], xb["beta"], S0=Sa, S_out=Sa,
                        per_key=False, out="f32")
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(x, False)
    check("o (segmented)", torch.cat([oa, ob], dim=3), o_ref, TOL["bf16"])
    check("S (segmented, in place)", Sa, S_ref, TOL["bf16"])
    check("o (full)", o_full, o_ref, TOL["bf16"])


def test_loop_independence():
    # The T-loop call sliced at loop tau equals a T=1 call on slice tau.
    w, x = _case("gdn_prefill", seed=4, T=3, B=2, H=2, L=96)
    o, S = run_prefill(x, per_key=False)
    for tau in range(3):
        xt = {k: (v[tau:tau + 1].contiguous() if isinstance(v, torch.Tensor) else v)
              for k, v in x.items()}
        ot, St = run_prefill(xt, per_key=False)
        assert torch.equal(ot, o[tau:tau + 1]) and torch.equal(St, S[tau:tau + 1])


# --- decode -----------------------------------------------------------------------------

@pytest.mark.parametrize("name,per_key", [("decode", False), ("kda_prefill", True),
                                          ("tiny_fp32", False)])
def test_decode_step(name, per_key):
    w = inputs.workload(name, T=2, B=3, H=4, L=1)
    dev = "cuda"
    g = torch.Generator().manual_seed(11)
    S = torch.randn((w.T, w.B, w.H, w.d, w.d), generator=g).to(dev) * 0.3
    x = to_device(inputs.make_decode_step(w, seed=1, step=0))
    S_gpu = S.clone()
    o = lt2.decode(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S_gpu, per_key=per_key,
                   out="f32")
    S_b = S.clone()
    o_b = lt2.decode(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S_b, per_key=per_key,
                     out="bf16")
    torch.cuda.synchronize()
    assert torch.equal(o_b, o.to(torch.bfloat16)) and torch.equal(S_b, S_gpu)
    o_ref, S_ref = oracle.decode_step(to_np(x["q"]), to_np(x["k"]), to_np(x["v"]),
                                      to_np(x["alpha"]), to_np(x["beta"]), to_np(S),
                                      per_key=per_key)
    tol = TOL[w.dtype]
    check("o", o, o_ref, tol)
    check("S", S_gpu, S_ref, tol)


@pytest.mark.parametrize("per_key", [False, True])
def test_decode_stepped_equals_prefill(per_key):
    name = "kda_prefill" if per_key else "gdn_prefill"
    w, x = _case(name, seed=9, T=2, B=2, H=2, L=40, s0="normal")
    o_pre, S_pre = run_prefill(x, per_key=per_key)
    S = x["S0"].clone()
    outs = []
    for t in range(w.L):
        a = x["alpha"][:, :, :, t]
        outs.append(lt2.decode(x["q"][:, :, :, t].contiguous(), x["k"][:, :, :, t].contiguous(),
                               x["v"][:, :, :, t].contiguous(), a.contiguous(),
                               x["beta"][:, :, :, t].contiguous(), S, per_key=per_key,
                               out="f32"))
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, dim=3)
    o_ref, S_ref = oracle_prefill(x, per_key)
    check("o decode-stepped", o_dec, o_ref, TOL["bf16"])
    check("S decode-stepped", S, S_ref, TOL["bf16"])
    check("o prefill", o_pre, o_ref, TOL["bf16"])
