"""The backward pass (lt2_gdr_backward) against the fp64 backward oracle of oracle/backward.py,
which is itself pinned by finite differences of the forward oracle.

Gradients of loss = sum(dO * o) + sum(dS_L * S_out) through the recurrence of "LT2 transformer
looped a tempo lineare", section "Sostituire il motore", displayed equation.  The kernel computes
in fp32 (its cross-column sums go through fp32 atomics, in no fixed order), so every gradient is
held to the library's fp32 bar, max|x - ref| / rms(ref) <= 1e-4, for fp32 and for bf16 inputs (the
oracle takes the same bf16 values).  Lengths cross the 64-token checkpoints of the kernel.
"""
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from oracle import backward as obw
from tests.gpu_util import TOL, check, to_np

pytestmark = pytest.mark.gpu


def _case(L, d, dtype, gate, seed, s0=True, dsl=True, T=2, H=2):
    w = inputs.workload("kda_prefill" if gate == "per_key" else "gdn_prefill", T=T, B=1, H=H, L=L, d=d,
                        dtype=dtype, s0="normal" if s0 else "zeros")
    x = inputs.make_inputs(w, seed=seed, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 100)
    x["dO"] = torch.randn(x["v"].shape, generator=g, device="cuda").to(x["v"].dtype)
    x["dS_L"] = torch.randn((T, 1, H, d, d), generator=g, device="cuda") if dsl else None
    return x


def _compare(x, per_key, order):
    g = lt2.backward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["dO"], S0=x.get("S0"), dS_L=x["dS_L"],
                     per_key=per_key, order=order)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    ref = obw.backward(*(to_np(x[n]) for n in ("q", "k", "v", "alpha", "beta", "dO")), S0=to_np(x.get("S0")),
                       dS_L=to_np(x["dS_L"]), per_key=per_key, order=order)
    for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dS0"):
        check(f"{n} ({order}, per_key={per_key})", g[n], ref[n], TOL["f32"])


GATES = [("scalar", "delta_first"), ("per_key", "delta_first"), ("per_key", "decay_first")]


@pytest.mark.parametrize("gate,order", GATES)
@pytest.mark.parametrize("L", [1, 64, 150])
def test_backward_fp32_matches_oracle(gate, order, L):
    _compare(_case(L, 32, "f32", gate, seed=L), gate == "per_key", order)


@pytest.mark.parametrize("gate,order", GATES)
def test_backward_bf16_d128_matches_oracle(gate, order):
    _compare(_case(130, 128, "bf16", gate, seed=7), gate == "per_key", order)


@pytest.mark.parametrize("gate,order", GATES)
def test_backward_fp32_d128_matches_oracle(gate, order):
    # fp32 inputs with d_k = 128: the compile-time instances whose workspace states move as float4
    _compare(_case(70, 128, "f32", gate, seed=5, T=1, H=2), gate == "per_key", order)


def test_backward_without_initial_state_or_final_gradient():
    _compare(_case(70, 64, "f32", "scalar", seed=3, s0=False, dsl=False), False, "delta_first")


def test_backward_odd_width():
    # d_v = 40: a full 32-column slice and a partial one
    w = inputs.workload("gdn_prefill", T=1, B=1, H=3, L=90, d=40, dtype="f32", s0="normal")
    x = inputs.make_inputs(w, seed=11, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(12)
    x["dO"] = torch.randn(x["v"].shape, generator=g, device="cuda")
    x["dS_L"] = torch.randn((1, 1, 3, 40, 40), generator=g, device="cuda")
    _compare(x, False, "delta_first")
