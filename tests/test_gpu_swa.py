"""The sliding-window mixer (lt2_swa_prefill) on both of its paths against the fp64 oracle of
oracle/swa.py, on the same seeded inputs.

"LT2 transformer looped a tempo lineare", section "Sostituire il motore": every token attends to
a window of the w most recent positions; section "Il giro trasforma il calcolo in contesto": over
T loops the window reaches back O(T w) tokens.

Tolerance, from the arithmetic: o_t is a convex combination of the v_s of its window, so every
error is measured against max|v| of the call (not rms(o), which shrinks as the window widens while
the first rows of a sequence stay as large as v).  The tensor-core kernel multiplies each
weight p_s = 2^(x_s - m) rounded to bf16 (relative error <= 2^-9) and divides by the fp32 sum of
the unrounded weights: o_t is off by sum_s w_s eps_s v_s with |eps_s| <= 2^-9, at most
2^-9 max|v|; fp32 accumulation and the approximate exp2 (relative error ~2^-22) add far less.
The bar, 2^-7 max|v|, leaves a margin of 4 over that bound; it is checked on an fp32 copy of o
(the bf16 output is checked to be that copy rounded to nearest).  The CUDA-core path computes in fp32 with expf and is
held to the library's fp32 bar, 1e-4 max|v|.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from oracle import swa as oswa
from tests.gpu_util import to_np

pytestmark = pytest.mark.gpu

TC, CC = lt2.LT2_ALGO_TENSOR_CORE, lt2.LT2_ALGO_CUDA_CORE
TOL_TC = 2.0 ** -7      # of max|v|
TOL_F32 = 1e-4     # of max|v|: the library's fp32 bar


def check(name, got, ref, v, tol):
    """max|got - ref| / max|v| <= tol."""
    err = np.abs(to_np(got) - ref).max() / np.abs(to_np(v)).max()
    assert np.isfinite(err) and err <= tol, f"{name}: max err {err:.3e} of max|v| > {tol:.1e}"
    return err


def _x(L, seed, T=2, B=1, H=2, d=128, dtype="bf16"):
    w = inputs.swa_workload("swa_prefill", T=T, B=B, H=H, L=L, d=d, dtype=dtype)
    return inputs.make_swa_inputs(w, seed=seed, device="cuda")


def _run(x, window, algo=lt2.LT2_ALGO_AUTO, out="f32", scale=None):
    o = lt2.swa_prefill(x["q"], x["k"], x["v"], window, scale=scale, algo=algo, out=out)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    return o


def _ref(x, window, scale=None):
    return oswa.prefill(to_np(x["q"]), to_np(x["k"]), to_np(x["v"]), window, scale=scale)


# L spans one and several 128-query blocks with ragged tails; windows below, at and across the
# 64-key block size, and wider than L
CASES = [(1, 1), (1, 7), (5, 3), (64, 64), (127, 1), (128, 65), (129, 128), (200, 2), (300, 63),
         (300, 64), (513, 200), (700, 700), (700, 5000), (1000, 333)]


@pytest.mark.parametrize("L,window", CASES)
def test_tensor_core_matches_oracle(L, window):
    x = _x(L, seed=L + window)
    check("o (tensor core)", _run(x, window, TC), _ref(x, window), x["v"], TOL_TC)


@pytest.mark.parametrize("L,window", [(1, 1), (77, 9), (300, 64), (513, 200)])
@pytest.mark.parametrize("d", [32, 100, 128, 256])
def test_cuda_core_fp32_is_exact(L, window, d):
    x = _x(L, seed=7 * L + d, d=d, dtype="f32")
    check("o (cuda core, fp32)", _run(x, window, CC), _ref(x, window), x["v"], TOL_F32)


@pytest.mark.parametrize("L,window", [(129, 17), (400, 128)])
def test_cuda_core_bf16_inputs(L, window):
    # bf16 inputs, fp32 arithmetic: the fp32 output at the fp32 bar (the oracle takes the same
    # bf16 values), the bf16 output that output rounded to nearest
    x = _x(L, seed=3 * L)
    o32 = _run(x, window, CC, out="f32")
    check("o (cuda core, bf16 in)", o32, _ref(x, window), x["v"], TOL_F32)
    o16 = _run(x, window, CC, out="bf16")
    assert o16.dtype == torch.bfloat16 and torch.equal(o16, o32.to(torch.bfloat16))


def test_auto_picks_a_path_for_every_shape():
    # bf16 d=128: the tensor-core kernel; fp32 or another width: the CUDA-core kernel
    for d, dtype in ((128, "bf16"), (64, "bf16"), (128, "f32")):
        x = _x(150, seed=d, d=d, dtype=dtype)
        tol = TOL_TC if (d, dtype) == (128, "bf16") else TOL_F32
        check(f"o (auto, d={d}, {dtype})", _run(x, 40, out="f32"), _ref(x, 40), x["v"], tol)


def test_forced_tensor_core_rejects_what_it_cannot_take():
    with pytest.raises(lt2.Lt2Error):
        lt2.swa_prefill(*(_x(64, 1, d=64)[n] for n in "qkv"), 8, algo=TC)
    with pytest.raises(lt2.Lt2Error):
        lt2.swa_prefill(*(_x(64, 1, dtype="f32")[n] for n in "qkv"), 8, algo=TC)


@pytest.mark.parametrize("L,window", [(300, 70), (1000, 128)])
def test_bf16_output_is_rounded_fp32_output(L, window):
    x = _x(L, seed=11)
    assert torch.equal(_run(x, window, TC, out="bf16"), _run(x, window, TC, out="f32").to(torch.bfloat16))


def test_window_one_returns_v_exactly():
    # a window of one token: the only weight is 1, o_t = v_t
    x = _x(333, seed=5)
    for algo in (TC, CC):
        assert torch.equal(_run(x, 1, algo, out="bf16"), x["v"])


def test_window_at_least_L_is_causal_attention():
    # w >= L: every window reaches back to token 0, the same result for every such w
    x = _x(260, seed=6)
    o1 = _run(x, 260, TC)
    assert torch.equal(o1, _run(x, 261, TC)) and torch.equal(o1, _run(x, 1 << 40, TC))
    check("o (w >= L)", o1, _ref(x, 260), x["v"], TOL_TC)


def test_explicit_scale_and_large_scores():
    # a non-default scale, and scores spread over hundreds (the running maximum is raised many
    # times inside a window and the output rescaled)
    x = _x(600, seed=8)
    check("o (scale 0.3)", _run(x, 150, TC, scale=0.3), _ref(x, 150, scale=0.3), x["v"], TOL_TC)
    big = {"q": (x["q"].float() * 6).to(torch.bfloat16), "k": (x["k"].float() * 6).to(torch.bfloat16), "v": x["v"]}
    check("o (large scores)", _run(big, 150, TC), _ref(big, 150), x["v"], TOL_TC)


def test_units_are_independent():
    # T, B and H all index independent units: each unit alone gives the same rows
    x = _x(200, seed=9, T=2, B=2, H=3)
    o = _run(x, 50, TC)
    one = {n: t[1:2, 0:1, 2:3].contiguous() for n, t in x.items()}
    assert torch.equal(o[1:2, 0:1, 2:3], _run(one, 50, TC))


def test_looped_receptive_field_on_the_gpu():
    # T loops chained (each loop's output is the next loop's values): a change of v at position p
    # reaches exactly the positions p .. p + T (w - 1), and leaves every other row bit-identical
    L, w, T, p = 400, 9, 4, 150
    x = _x(L, seed=10, T=1, H=1)

    def looped(v0):
        y = v0
        for _ in range(T):
            y = _run({"q": x["q"], "k": x["k"], "v": y}, w, TC, out="bf16")
        return y
    v2 = x["v"].clone()
    v2[..., p, :] += 100.0
    diff = (looped(x["v"]).float() - looped(v2).float()).abs().amax(dim=-1).flatten().cpu().numpy()
    reach = p + T * (w - 1)
    assert np.all(diff[:p] == 0) and np.all(diff[reach + 1:] == 0)
    assert diff[p] > 0 and diff[reach] > 0
    assert np.mean(diff[p:reach + 1] > 0) > 0.9


def test_full_size_sampled_rows():
    # the swa_prefill workload (T4 B4 H16 L8192 d128, w=512) in one call; in one unit of every loop,
    # 96 consecutive rows at the start, the middle and the end checked against the oracle (each
    # row's window taken whole)
    w = inputs.swa_workload("swa_prefill")
    x = inputs.make_swa_inputs(w, seed=0, device="cuda")
    o = _run(x, w.window, out="f32")
    rng = np.random.default_rng(4)
    for t in range(w.T):
        b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
        for r0 in (0, w.L // 2 - 48, w.L - 96):
            s0 = max(0, r0 - w.window + 1)
            sl = slice(s0, r0 + 96)
            ref = oswa.prefill(*(to_np(x[n][t, b, h, sl]) for n in "qkv"), w.window)[r0 - s0:]
            check(f"o (loop {t}, rows {r0}..)", o[t, b, h, r0:r0 + 96], ref, x["v"][t, b, h, sl], TOL_TC)
