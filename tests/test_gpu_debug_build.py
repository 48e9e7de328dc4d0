"""The debug build of the library (liblt2gdr_debug.so, include/lt2_gdr_debug.h) on the GPU.

- Its device-side checks (TMA coordinates, shared-memory tiles, TMEM columns) hold on small and
  ragged problems of both tensor-core prefills: no LT2_ERR_DEVICE_CHECK, and the results match
  the oracle.
- A bounded wait that runs out is reported, not hung on: the TMA producer is made to stop before
  one chunk, the waits for that chunk's copies give up after the debug build's short bound, the
  kernel records LT2_ERR_DEVICE_TIMEOUT, drains what it has in flight, frees its tensor memory
  and returns.  The status is read once and then cleared, and the next call (same process, same
  context) is correct.  Nothing traps and nothing waits without a bound.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import build as lbuild
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill

pytestmark = pytest.mark.gpu

KERNEL = {"scalar": 0, "per_key": 1}         # lt2_debug_kernel


@pytest.fixture(scope="module")
def D():
    if lbuild.needs_build(debug=True):
        lbuild.build(debug=True)
    L = lt2.load_library(lbuild.DEBUG_LIB)
    assert 0 < L.lt2_debug_wait_timeout_ns() <= 100_000_000
    yield L
    for k in KERNEL.values():
        L.lt2_debug_set_skip_chunk(k, -1)


def _inputs(gate, L, seed, H=2):
    w = inputs.workload("kda_prefill" if gate == "per_key" else "gdn_prefill", T=1, B=1, H=H, L=L,
                        s0="normal")
    return inputs.make_inputs(w, seed=seed, device="cuda")


def _prefill(lib, x, gate, out="f32"):
    """One tensor-core prefill through `lib`; returns (o, S_T, launch status)."""
    per_key = gate == "per_key"
    dims = lt2._dims_from(x["q"], x["v"], x["alpha"], per_key, lt2.LT2_ALGO_TENSOR_CORE, out)
    o = torch.empty(x["v"].shape, dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    S = torch.empty(tuple(x["q"].shape[:3]) + (128, 128), dtype=torch.float32, device="cuda")
    st = lib.lt2_gdr_prefill(ctypes.byref(dims), x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                             x["alpha"].data_ptr(), x["beta"].data_ptr(), x["S0"].data_ptr(), o.data_ptr(),
                             S.data_ptr(), None, 0, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return o, S, st


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("L", [1, 63, 65, 200])
def test_debug_checks_hold_and_results_match(D, gate, L):
    # parity on the fp32 output; the bf16 output (TMA-stored) is exactly the fp32 one rounded
    x = _inputs(gate, L, seed=L)
    o32, S, st = _prefill(D, x, gate, "f32")
    assert st == lt2.LT2_OK
    assert D.lt2_gdr_last_device_error() == lt2.LT2_OK
    o_ref, S_ref = oracle_prefill(x, gate == "per_key")
    check("o", o32, o_ref, TOL["bf16"])
    check("S_T", S, S_ref, TOL["bf16"])
    o16, S16, st = _prefill(D, x, gate, "bf16")
    assert st == lt2.LT2_OK
    assert D.lt2_gdr_last_device_error() == lt2.LT2_OK
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S)


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("skip", [0, 2])
def test_a_wait_that_runs_out_is_reported_then_cleared(D, gate, skip):
    x = _inputs(gate, 300, seed=11)
    assert D.lt2_debug_set_skip_chunk(KERNEL[gate], skip) == lt2.LT2_OK
    try:
        _, _, st = _prefill(D, x, gate)
        assert st == lt2.LT2_OK                          # the launch itself succeeded
        assert D.lt2_gdr_last_device_error() == lt2.LT2_ERR_DEVICE_TIMEOUT
        assert D.lt2_gdr_last_device_error() == lt2.LT2_OK   # read once, then cleared
    finally:
        assert D.lt2_debug_set_skip_chunk(KERNEL[gate], -1) == lt2.LT2_OK
    # the same call again, in the same context: the kernel freed its tensor memory and the
    # status word is clean, so it runs to the end and is right
    o, S, st = _prefill(D, x, gate)
    assert st == lt2.LT2_OK and D.lt2_gdr_last_device_error() == lt2.LT2_OK
    o_ref, S_ref = oracle_prefill(x, gate == "per_key")
    check("o after the timeout", o, o_ref, TOL["bf16"])
    check("S_T after the timeout", S, S_ref, TOL["bf16"])
    # and the product library, in the same process, is unaffected
    o2, S2 = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x["S0"],
                         per_key=gate == "per_key", algo=lt2.LT2_ALGO_TENSOR_CORE, out="f32")
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    check("o (product library)", o2, o_ref, TOL["bf16"])


def test_injection_arguments_are_checked(D):
    assert D.lt2_debug_set_skip_chunk(5, 0) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert D.lt2_debug_set_skip_chunk(0, -2) == lt2.LT2_ERR_INVALID_ARGUMENT
