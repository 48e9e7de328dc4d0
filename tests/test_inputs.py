"""The seeded input recipe (CPU): the one module the CUDA library and the oracle share draws
exactly what its docstring states, deterministically."""
import math

import pytest
import torch

from gated_delta_rule_looped_b200 import inputs


def test_workload_sizes():
    w = {n: inputs.workload(n) for n in inputs.WORKLOADS}
    assert (w["gdn_prefill"].T, w["gdn_prefill"].B, w["gdn_prefill"].H, w["gdn_prefill"].L) == (4, 4, 16, 8192)
    assert (w["kda_prefill"].T, w["kda_prefill"].B, w["kda_prefill"].H, w["kda_prefill"].L) == (4, 2, 16, 16384)
    assert (w["decode"].T, w["decode"].B, w["decode"].H, w["decode"].history) == (4, 256, 16, 4096)
    assert (w["long_gdn"].T, w["long_gdn"].B, w["long_gdn"].H, w["long_gdn"].L) == (8, 1, 32, 65536)
    assert w["kda_prefill"].gate == "per_key" and w["gdn_prefill"].gate == "scalar"
    assert all(x.d == 128 for n, x in w.items() if n != "tiny_fp32") and w["tiny_fp32"].d == 32
    assert inputs.workload("gdn_prefill", L=100).L == 100


@pytest.mark.parametrize("name", ["gdn_prefill", "kda_prefill", "tiny_fp32"])
def test_shapes_ranges_and_unit_rows(name):
    w = inputs.workload(name, T=2, B=2, H=3, L=50, s0="normal")
    x = inputs.make_inputs(w, seed=5)
    shp = (2, 2, 3, 50, w.d)
    assert x["q"].shape == shp and x["k"].shape == shp and x["v"].shape == shp
    assert x["q"].dtype == w.torch_dtype
    a = x["alpha"]
    assert a.shape == (shp if w.gate == "per_key" else shp[:-1]) and a.dtype == torch.float32
    assert x["beta"].shape == shp[:-1] and x["S0"].shape == (2, 2, 3, w.d, w.d)
    assert ((a > 0) & (a <= 1)).all()
    if name == "tiny_fp32":
        assert (a >= 0.9).all()
    else:
        assert (a > math.exp(-math.log1p(math.exp(8.0)) * 0.1)).all()   # exp(-softplus(x) 0.1), |x| < 8
    b = x["beta"]
    assert ((b > 0) & (b < 1)).all()
    # q, k unit norm per (token, head), up to the rounding of their dtype
    tol = 1e-5 if w.dtype == "f32" else 2 ** -7
    for n in ("q", "k"):
        norms = x[n].float().norm(dim=-1)
        assert (norms - 1).abs().max() <= tol


def test_overwrite_subset():
    w = inputs.workload("long_gdn", T=2, B=3, H=2, L=700)
    x = inputs.make_inputs(w, seed=2, q_equals_k_on_subset=True)
    sub = x["subset"]
    assert sub.shape == (2, 3, 700)
    assert (sub.sum(dim=-1) == round(0.01 * 700)).all()
    m = sub[:, :, None, :].expand(2, 3, 2, 700)
    assert (x["alpha"][m] == 1).all() and (x["beta"][m] == 1).all()
    assert torch.equal(x["q"][m], x["k"][m])
    assert (x["alpha"][~m] < 1).all()


def test_deterministic_per_seed():
    w = inputs.workload("kda_prefill", T=1, B=1, H=2, L=40)
    a, b, c = (inputs.make_inputs(w, seed=s) for s in (3, 3, 4))
    for n in ("q", "k", "v", "alpha", "beta"):
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])


def test_decode_step_shapes():
    w = inputs.workload("kda_prefill", T=2, B=3, H=4, L=1)
    x = inputs.make_decode_step(w, seed=1, step=0)
    assert x["q"].shape == (2, 3, 4, 128) and x["alpha"].shape == (2, 3, 4, 128)
    assert x["beta"].shape == (2, 3, 4)
    y = inputs.make_decode_step(w, seed=1, step=1)
    assert not torch.equal(x["q"], y["q"])
