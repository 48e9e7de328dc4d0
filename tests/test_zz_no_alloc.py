"""The allocation-free backward entry point, lt2_gdr_backward_static, against lt2_gdr_backward.

Some callers cannot allocate device memory: their device memory is handed out entirely by a host
application's or framework's own allocator, or they serve requests and must not call cudaMalloc,
which can block the whole device.  lt2_gdr_backward_static gives them the backward pass with its
scratch in a fixed array inside the library instead of a caller-provided workspace.  This file
checks, through the C ABI, that two calls in a row (the second on new inputs, over the scratch the
first one left behind) give the gradients of the workspace entry point within the library's fp32
bar, and that a problem too large for the array is refused.  It is collected last on purpose.
"""
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


def _case(seed, T=2, H=3, L=150, d=64, dtype="bf16"):
    w = inputs.workload("gdn_prefill", T=T, B=1, H=H, L=L, d=d, dtype=dtype, s0="normal")
    x = inputs.make_inputs(w, seed=seed, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    x["dO"] = torch.randn(x["v"].shape, generator=g, device="cuda").to(x["v"].dtype)
    x["dS_L"] = torch.randn((T, 1, H, d, d), generator=g, device="cuda")
    dims = lt2.make_dims(T, 1, H, L, d, d, lt2.LT2_DTYPE_BF16 if dtype == "bf16" else lt2.LT2_DTYPE_F32,
                         lt2.LT2_GATE_SCALAR)
    return x, dims


def _grads(x):
    f32 = dict(dtype=torch.float32, device="cuda")
    return {"dq": torch.empty(x["q"].shape, **f32), "dk": torch.empty(x["q"].shape, **f32),
            "dv": torch.empty(x["v"].shape, **f32), "dalpha": torch.empty(x["alpha"].shape, **f32),
            "dbeta": torch.empty(x["beta"].shape, **f32), "dS0": torch.empty(x["dS_L"].shape, **f32)}


def _inputs(x):
    return (x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], x["dO"], x["dS_L"])


def test_static_scratch_matches_workspace_entry_on_two_calls_in_a_row():
    for seed, dtype in ((1, "bf16"), (2, "f32")):
        x, dims = _case(seed, dtype=dtype)
        ref = _grads(x)
        ws_bytes = lt2.lt2_gdr_backward_workspace_bytes(dims)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        st = lt2.lt2_gdr_backward(dims, *_inputs(x), *(ref[n] for n in NAMES), ws, ws_bytes)
        assert st == lt2.LT2_OK
        got = _grads(x)
        st = lt2.lt2_gdr_backward_static(dims, *_inputs(x), *(got[n] for n in NAMES))
        assert st == lt2.LT2_OK
        torch.cuda.synchronize()
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        for n in NAMES:
            check(f"{n} (static scratch, call {seed})", got[n], ref[n].double().cpu().numpy(), TOL["f32"])


def test_too_large_for_the_static_scratch_is_refused():
    # 6 units of 8,192 tokens at d = 128 need more than the 64 MiB array holds
    dims = lt2.make_dims(1, 1, 6, 8192, 128, 128, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)
    assert lt2.lt2_gdr_backward_workspace_bytes(dims) > 64 << 20
    fake = [1 << 40] * 14                         # never touched: the call returns before any launch
    assert lt2.lt2_gdr_backward_static(dims, *fake) == lt2.LT2_ERR_WORKSPACE
