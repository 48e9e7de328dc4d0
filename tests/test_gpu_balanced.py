"""The scalar tensor-core prefill's balanced schedule (more units than SMs, a workspace, S_out):
one CTA per SM takes an equal share of all units' chunks, and a unit split between two CTAs hands
its state over through S_out.  Its results must be those of the one-unit-per-CTA launches bit
for bit (same chunk arithmetic, the handed-over state is the fp32 state), and the oracle's.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, oracle_prefill

pytestmark = pytest.mark.gpu


def _call(x, dims, o, S, S0, ws):
    nbytes = lt2.lt2_gdr_prefill_workspace_bytes(dims) if ws is not None else 0
    st = lt2.lt2_gdr_prefill(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0, o, S, ws, nbytes)
    torch.cuda.synchronize()
    assert st == lt2.LT2_OK and lt2.lt2_gdr_last_device_error() == lt2.LT2_OK


@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("L", [200, 64, 333])
def test_balanced_equals_per_unit_launches(L, out):
    # T2 B2 H40: 160 units on 148 SMs, split units at several chunk positions
    w = inputs.workload("gdn_prefill", T=2, B=2, H=40, L=L, s0="normal")
    x = inputs.make_inputs(w, seed=L, device="cuda")
    dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR,
                         out_dtype=lt2.LT2_OUT_BF16 if out == "bf16" else lt2.LT2_OUT_F32)
    odt = torch.bfloat16 if out == "bf16" else torch.float32
    nbytes = lt2.lt2_gdr_prefill_workspace_bytes(dims)
    assert nbytes >= 4 * w.T * w.B * w.H
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    res = []
    for use_ws in (True, False):
        o = torch.full(x["v"].shape, 3.0, dtype=odt, device="cuda")
        S = torch.full((w.T, w.B, w.H, 128, 128), 5.0, device="cuda")
        _call(x, dims, o, S, x["S0"], ws if use_ws else None)
        res.append((o, S))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    if out == "bf16":
        return                      # (parity on the fp32 output; bf16 is its rounding, tested elsewhere)
    units = [(0, 0, 0), (1, 1, 39), (0, 1, 17), (1, 0, 25)]
    o_ref, S_ref = oracle_prefill(x, False, units=units)
    o_sel = torch.stack([res[0][0][u] for u in units])
    S_sel = torch.stack([res[0][1][u] for u in units])
    check("o (balanced)", o_sel, o_ref, TOL["bf16"])
    check("S_T (balanced)", S_sel, S_ref, TOL["bf16"])


def test_balanced_in_place_resume_and_fused_steps():
    # S0 == S_out (in place) with the fused prologue and output gate, 150 units
    w = inputs.workload("gdn_prefill", T=1, B=3, H=50, L=150, s0="normal")
    r = inputs.make_raw_inputs(w, seed=5, device="cuda")
    outs = []
    for use_ws in (True, False):
        S = r["S0"].clone()
        o = torch.empty(r["v"].shape, dtype=torch.bfloat16, device="cuda")
        dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)
        fused = lt2.make_fused(True, True, 0.1, r["z"])
        nbytes = lt2.lt2_gdr_prefill_workspace_bytes(dims) if use_ws else 0
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda") if use_ws else None
        st = lt2.lt2_gdr_prefill_fused(dims, fused, r["q"], r["k"], r["v"], r["a"], r["b"], S, o, S, ws, nbytes)
        torch.cuda.synchronize()
        assert st == lt2.LT2_OK and lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        outs.append((o, S))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_short_workspace_is_refused():
    w = inputs.workload("gdn_prefill", T=1, B=1, H=150, L=64)
    x = inputs.make_inputs(w, seed=1, device="cuda")
    dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)
    nbytes = lt2.lt2_gdr_prefill_workspace_bytes(dims)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = torch.empty(x["v"].shape, dtype=torch.bfloat16, device="cuda")
    S = torch.empty((1, 1, 150, 128, 128), device="cuda")
    st = lt2.lt2_gdr_prefill(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], None, o, S, ws, nbytes - 16)
    assert st == lt2.LT2_ERR_WORKSPACE


def test_balanced_from_zero_states_and_without_final_state_request():
    # S0 = NULL (zero states); the balanced schedule needs S_out, which lt2.prefill always passes
    w = inputs.workload("gdn_prefill", T=3, B=1, H=60, L=129)
    x = inputs.make_inputs(w, seed=6, device="cuda")
    dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR,
                         out_dtype=lt2.LT2_OUT_F32)
    nbytes = lt2.lt2_gdr_prefill_workspace_bytes(dims)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    res = []
    for use_ws in (True, False):
        o = torch.empty(x["v"].shape, dtype=torch.float32, device="cuda")
        S = torch.empty((w.T, w.B, w.H, 128, 128), device="cuda")
        _call(x, dims, o, S, None, ws if use_ws else None)
        res.append((o, S))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    # without S_out the call runs one unit per CTA and gives the same outputs
    o = torch.empty(x["v"].shape, dtype=torch.float32, device="cuda")
    _call(x, dims, o, None, None, ws)
    assert torch.equal(o, res[0][0])
    units = [(0, 0, 0), (2, 0, 59), (1, 0, 31)]
    x0 = dict(x, S0=None)
    o_ref, S_ref = oracle_prefill(x0, False, units=units)
    check("o (balanced, zero states)", torch.stack([res[0][0][u] for u in units]), o_ref, TOL["bf16"])
    check("S_T (balanced, zero states)", torch.stack([res[0][1][u] for u in units]), S_ref, TOL["bf16"])

