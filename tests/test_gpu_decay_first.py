"""GPU parity of the decay-first per-key order against the fp64 oracle.

The per-key equation of "LT2 transformer looped a tempo lineare" (section "Sostituire il
motore") prints A_t = Diag(alpha_t)(I - beta_t k_t k_t^T); the other reading of the same symbols,
A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), applies the decay before the delta step.  Every path
that takes per-key gating (the tensor-core chunked prefill with its token-by-token chunks, the
CUDA-core prefill and the decode step) runs it under LT2_GATE_PER_KEY_DECAY_FIRST, checked here
against the oracle's decay-first order.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
import oracle
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill, run_prefill, to_device, to_np

pytestmark = pytest.mark.gpu

TC = lt2.LT2_ALGO_TENSOR_CORE
CC = lt2.LT2_ALGO_CUDA_CORE
DF = "decay_first"


def _run(x, algo, tol):
    o, S = run_prefill(x, per_key=True, algo=algo, order=DF)
    o_ref, S_ref = oracle_prefill(x, True, order=DF)
    check("o", o, o_ref, tol)
    check("S_T", S, S_ref, tol)
    return o


@pytest.mark.parametrize("L", [1, 31, 32, 33, 100, 333])
def test_decay_first_tensor_core_lengths(L):
    w = inputs.workload("kda_prefill", T=2, B=1, H=2, L=L, s0="normal")
    _run(to_device(inputs.make_inputs(w, seed=500 + L)), TC, TOL["bf16"])


def test_decay_first_tensor_core_workload_distribution():
    w = inputs.workload("kda_prefill", T=2, B=2, H=3, L=2048)
    _run(to_device(inputs.make_inputs(w, seed=12)), TC, TOL["bf16"])


@pytest.mark.parametrize("power", [6.0, 40.0])
def test_decay_first_tensor_core_strong_decay(power):
    # some chunks (alpha^6) or all of them (alpha^40) beyond the fp16 tile range: those run
    # token by token in the kernel, in the same order
    w = inputs.workload("kda_prefill", T=1, B=2, H=2, L=640, s0="normal")
    x = inputs.make_inputs(w, seed=42)
    x["alpha"] = x["alpha"].double().pow(power).float()
    _run(to_device(x), TC, TOL["bf16"])


def test_decay_first_tensor_core_resets():
    w = inputs.workload("kda_prefill", T=1, B=1, H=3, L=300, s0="normal")
    x = inputs.make_inputs(w, seed=44)
    a = x["alpha"].clone()
    a[..., 37, 5] = 0.0
    a[..., 130, :] = 0.0
    x["alpha"] = a
    _run(to_device(x), TC, TOL["bf16"])


@pytest.mark.parametrize("name,tol", [("kda_prefill", TOL["bf16"]), ("tiny_fp32", TOL["f32"])])
def test_decay_first_cuda_core(name, tol):
    over = dict(T=2, B=1, H=2, L=77, s0="normal")
    w = inputs.workload(name, **over)
    x = inputs.make_inputs(w, seed=61)
    if x["alpha"].dim() == 4:                      # tiny_fp32 draws a scalar gate: make it per key
        g = torch.Generator().manual_seed(5)
        x["alpha"] = (x["alpha"][..., None] * (0.9 + 0.1 * torch.rand(x["q"].shape, generator=g))).contiguous()
    _run(to_device(x), CC, tol)


def test_decay_first_paths_agree_and_differ_from_delta_first():
    w = inputs.workload("kda_prefill", T=1, B=2, H=2, L=400, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=7))
    o_tc = _run(x, TC, TOL["bf16"])
    o_cc, _ = run_prefill(x, per_key=True, algo=CC, order=DF)
    o_ref, _ = oracle_prefill(x, True, order=DF)
    assert check("o cuda-core", o_cc, o_ref, 1e-4) < check("o tensor-core", o_tc, o_ref, TOL["bf16"])
    # the flag reaches the kernels: the printed order gives a different result
    o_lit, _ = run_prefill(x, per_key=True, algo=TC)
    assert oracle.rel_max_err(to_np(o_lit), o_ref) > 3 * TOL["bf16"]


def test_decay_first_decode_step():
    w = inputs.workload("kda_prefill", T=2, B=3, H=4, L=1)
    g = torch.Generator().manual_seed(13)
    S = torch.randn((w.T, w.B, w.H, w.d, w.d), generator=g).cuda() * 0.3
    x = to_device(inputs.make_decode_step(w, seed=2, step=0))
    S_gpu = S.clone()
    o = lt2.decode(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S_gpu, per_key=True, out="f32",
                   order=DF)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.decode_step(to_np(x["q"]), to_np(x["k"]), to_np(x["v"]), to_np(x["alpha"]),
                                      to_np(x["beta"]), to_np(S), per_key=True, order=DF)
    check("o", o, o_ref, TOL["bf16"])
    check("S", S_gpu, S_ref, TOL["bf16"])


def test_decay_first_decode_stepped_equals_prefill():
    w = inputs.workload("kda_prefill", T=2, B=2, H=2, L=40, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=19))
    S = x["S0"].clone()
    outs = []
    for t in range(w.L):
        outs.append(lt2.decode(x["q"][:, :, :, t].contiguous(), x["k"][:, :, :, t].contiguous(),
                               x["v"][:, :, :, t].contiguous(), x["alpha"][:, :, :, t].contiguous(),
                               x["beta"][:, :, :, t].contiguous(), S, per_key=True, out="f32", order=DF))
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(x, True, order=DF)
    check("o decode-stepped", torch.stack(outs, dim=3), o_ref, TOL["bf16"])
    check("S decode-stepped", S, S_ref, TOL["bf16"])


def test_decay_first_overwrite_invariant_on_gpu():
    # beta = 1 and unit keys: reading with q = k returns v for any per-key decay (decay-first
    # order only), on the fp32 CUDA-core path where the check is tight
    w = inputs.workload("tiny_fp32", T=1, B=1, H=2, L=50, s0="normal")
    x = inputs.make_inputs(w, seed=3)
    g = torch.Generator().manual_seed(8)
    x["alpha"] = (0.5 + 0.5 * torch.rand(x["q"].shape, generator=g)).contiguous()
    x["beta"] = torch.ones_like(x["beta"])
    x["q"] = x["k"].clone()
    x = to_device(x)
    o, _ = run_prefill(x, per_key=True, algo=CC, order=DF)
    v = to_np(x["v"])
    assert np.max(np.abs(to_np(o) - v)) <= 1e-4 * np.max(np.abs(v))
