"""GPU parity of the tensor-core (tcgen05/TMA) chunked prefill against the fp64 oracle:
ragged lengths around the 64-token chunk, several chunks, non-zero initial state, the
overwrite positions of the long-context workload, and agreement with the CUDA-core path."""
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill, run_prefill, to_device

pytestmark = pytest.mark.gpu

TC = lt2.LT2_ALGO_TENSOR_CORE


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 130, 333, 1000])
def test_tc_lengths(L):
    w = inputs.workload("gdn_prefill", T=2, B=1, H=2, L=L, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=100 + L))
    o, S = run_prefill(x, per_key=False, algo=TC)
    o_ref, S_ref = oracle_prefill(x, False)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("name", ["gdn_prefill", "long_gdn"])
def test_tc_workload_distributions(name):
    w = inputs.workload(name, T=2, B=2, H=3, L=2048)
    x = to_device(inputs.make_inputs(w, seed=7))
    o, S = run_prefill(x, per_key=False, algo=TC)
    o_ref, S_ref = oracle_prefill(x, False)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])


def test_tc_overwrite_invariant_with_q_equal_k():
    # At the alpha = beta = 1 positions with q_t := k_t, o_t = S_t^T k_t must equal v_t up to
    # (1 - |k_t|^2) (S_{t-1}^T k_t - v_t): k_t is unit-norm only up to its bf16 rounding.
    w = inputs.workload("long_gdn", T=1, B=1, H=4, L=4096)
    x = to_device(inputs.make_inputs(w, seed=5, q_equals_k_on_subset=True))
    o, S = run_prefill(x, per_key=False, algo=TC)
    o_ref, _ = oracle_prefill(x, False)
    check("o", o, o_ref, TOL["bf16"])
    m = x["subset"][0, 0]
    v = x["v"][0, 0][:, m].float()
    k = x["k"][0, 0][:, m].float()
    slack = (1 - (k * k).sum(-1)).abs().max().item()
    err = (o[0, 0][:, m] - v).abs().max().item() / v.pow(2).mean().sqrt().item()
    assert err <= TOL["bf16"] + 10 * slack, err


def test_tc_matches_cuda_core_path():
    w = inputs.workload("gdn_prefill", T=1, B=2, H=2, L=777, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=3))
    o_tc, S_tc = run_prefill(x, per_key=False, algo=TC)
    o_cc, S_cc = run_prefill(x, per_key=False, algo=lt2.LT2_ALGO_CUDA_CORE)
    o_ref, S_ref = oracle_prefill(x, False)
    # the fp32 CUDA-core path is far closer to the oracle; both within the bar
    assert check("o cuda-core", o_cc, o_ref, 1e-4) < check("o tensor-core", o_tc, o_ref, TOL["bf16"])
    check("S tensor-core", S_tc, S_ref, TOL["bf16"])


def test_tc_in_place_state_and_no_final_state():
    w = inputs.workload("gdn_prefill", T=2, B=1, H=2, L=200, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=8))
    o_ref, S_ref = oracle_prefill(x, False)
    S = x["S0"].clone()
    o, _ = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=S, S_out=S, per_key=False,
                       algo=TC, out="f32")
    torch.cuda.synchronize()
    check("o (S0 == S_out)", o, o_ref, TOL["bf16"])
    check("S (in place)", S, S_ref, TOL["bf16"])
    # S_out = NULL through the raw ABI
    dims = lt2.make_dims(2, 1, 2, 200, 128, 128, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR, TC,
                         lt2.LT2_OUT_F32)
    o2 = torch.empty_like(o)
    st = lt2.lt2_gdr_prefill(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], o2, None)
    torch.cuda.synchronize()
    assert st == lt2.LT2_OK and lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    assert torch.equal(o2, o)


@pytest.mark.parametrize("power", [30.0, 3.0])
def test_tc_strong_decay(power):
    # alpha^30 gives a chunk decay far below e^-80, where e^{-G} is not representable and the
    # chunk matrices take the unfactored e^{G_r - G_s}; alpha^3 mixes both kinds of chunk.
    w = inputs.workload("gdn_prefill", T=1, B=1, H=3, L=450, s0="normal")
    x = inputs.make_inputs(w, seed=21)
    x["alpha"] = x["alpha"].double().pow(power).float()
    x = to_device(x)
    o, S = run_prefill(x, per_key=False, algo=TC)
    o_ref, S_ref = oracle_prefill(x, False)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])
