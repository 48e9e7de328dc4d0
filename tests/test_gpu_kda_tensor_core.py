"""GPU parity of the per-key (KDA-style) tensor-core chunked prefill against the fp64 oracle:
ragged lengths around the 32-token chunk, the workload's gate distribution, a non-zero initial
state, chunks whose per-key decay is beyond the range of the fp16 Gram tiles (those run token by
token inside the kernel), alpha = 0 resets, in-place resume, and agreement with the CUDA-core
path."""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill, run_prefill, to_device

pytestmark = pytest.mark.gpu

TC = lt2.LT2_ALGO_TENSOR_CORE
CHUNK = 32
# The Gram tiles of a chunk carry e^{+-(G - G_31/2)} and must stay within [2^-14, 2^14]: for
# alpha in (0, 1] that holds while every key's chunk decay P_31 is at least 2^-28.
P31_MIN = 2.0 ** -28


def _chunk_kinds(alpha, L):
    """(in-range chunks, exact chunks) over all units of an alpha tensor [..., L, d]."""
    a = alpha.double().reshape(-1, L, alpha.shape[-1])
    n_in = n_ex = 0
    for c0 in range(0, L, CHUNK):
        p31 = a[:, c0:c0 + CHUNK, :].prod(dim=1)          # [units, d]
        ok = (p31 >= P31_MIN).all(dim=1)
        n_in += int(ok.sum())
        n_ex += int((~ok).sum())
    return n_in, n_ex


def _run(x):
    o, S = run_prefill(x, per_key=True, algo=TC)
    o_ref, S_ref = oracle_prefill(x, True)
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 64, 65, 100, 333])
def test_kda_tc_lengths(L):
    w = inputs.workload("kda_prefill", T=2, B=1, H=2, L=L, s0="normal")
    _run(to_device(inputs.make_inputs(w, seed=300 + L)))


def test_kda_tc_workload_distribution():
    w = inputs.workload("kda_prefill", T=2, B=2, H=3, L=2048)
    x = inputs.make_inputs(w, seed=11)
    assert _chunk_kinds(x["alpha"], w.L)[1] == 0          # the recipe stays in range
    _run(to_device(x))


@pytest.mark.parametrize("power", [6.0, 40.0])
def test_kda_tc_strong_decay(power):
    # alpha^6: some chunks in range, most beyond it (mixed); alpha^40: all beyond it
    w = inputs.workload("kda_prefill", T=1, B=2, H=2, L=640, s0="normal")
    x = inputs.make_inputs(w, seed=41)
    x["alpha"] = x["alpha"].double().pow(power).float()
    n_in, n_ex = _chunk_kinds(x["alpha"], w.L)
    assert n_ex > 0
    if power == 6.0:
        assert n_in > 0
    _run(to_device(x))


def test_kda_tc_resets():
    # alpha = 0 on some (token, key) entries wipes those state rows; a chunk holding one runs
    # token by token
    w = inputs.workload("kda_prefill", T=1, B=1, H=3, L=300, s0="normal")
    x = inputs.make_inputs(w, seed=43)
    a = x["alpha"].clone()
    a[..., 37, 5] = 0.0
    a[..., 130, :] = 0.0
    a[0, 0, 1, 201, 64:] = 0.0
    x["alpha"] = a
    n_in, n_ex = _chunk_kinds(a, w.L)
    assert n_in > 0 and n_ex > 0
    _run(to_device(x))


def test_kda_tc_matches_cuda_core_path():
    w = inputs.workload("kda_prefill", T=1, B=2, H=2, L=777, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=5))
    o_tc, S_tc = run_prefill(x, per_key=True, algo=TC)
    o_cc, S_cc = run_prefill(x, per_key=True, algo=lt2.LT2_ALGO_CUDA_CORE)
    o_ref, S_ref = oracle_prefill(x, True)
    assert check("o cuda-core", o_cc, o_ref, 1e-4) < check("o tensor-core", o_tc, o_ref, TOL["bf16"])
    check("S tensor-core", S_tc, S_ref, TOL["bf16"])


def test_kda_tc_in_place_resume_and_bf16_output():
    w = inputs.workload("kda_prefill", T=2, B=1, H=2, L=150, s0="normal")
    x = to_device(inputs.make_inputs(w, seed=9))
    o_ref, S_ref = oracle_prefill(x, True)
    S = x["S0"].clone()
    o32, _ = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=S, S_out=S, per_key=True,
                         algo=TC, out="f32")
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    check("o (S0 == S_out)", o32, o_ref, TOL["bf16"])
    check("S (in place)", S, S_ref, TOL["bf16"])
    o16, _ = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x["S0"], per_key=True, algo=TC,
                         out="bf16")
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))


@pytest.mark.parametrize("order", ["delta_first", "decay_first"])
def test_kda_tc_alpha_above_one(order):
    # mild growth (alpha > 1 on a few tokens, the state and every tile staying well inside fp16)
    # runs on the tensor cores, in either order
    w = inputs.workload("kda_prefill", T=1, B=1, H=2, L=200, s0="normal")
    x = inputs.make_inputs(w, seed=47)
    a = x["alpha"].clone()
    a[..., 64:72, :] = 1.5
    a[..., 130:140, :7] = 1.02
    x["alpha"] = a
    x = to_device(x)
    o, S = run_prefill(x, per_key=True, algo=TC, order=order)
    o_ref, S_ref = oracle_prefill(x, True, order=order)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    check("o", o, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])
