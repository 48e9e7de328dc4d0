"""Parity at the workloads' full sizes, in the configuration the benchmark times (all T loops
in one call, bf16 q/k/v, fp32 state), on sampled (loop, batch, head) units that the fp64 oracle
recomputes one by one.  o is checked in its fp32 form against the oracle (<= 2e-2 of rms), and
the bf16 output of the same call is checked to be exactly that fp32 result rounded."""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
import oracle
from gated_delta_rule_looped_b200 import inputs
from tests.gpu_util import TOL, check, to_np

pytestmark = pytest.mark.gpu


def _units(w, n, seed):
    """The first and last head-units, one unit of every loop (each loop is its own launch, and
    the later launches run on the second wave of CTAs), then random units up to n."""
    rng = np.random.default_rng(seed)
    picks = {(w.T - 1, w.B - 1, w.H - 1), (0, 0, 0)}
    for tau in range(w.T):
        picks.add((tau, int(rng.integers(w.B)), int(rng.integers(w.H))))
    while len(picks) < n:
        picks.add((int(rng.integers(w.T)), int(rng.integers(w.B)), int(rng.integers(w.H))))
    return sorted(picks)


def _check_sampled(x, o32, S, units, per_key, S0=None, order="delta_first"):
    sel = lambda t: torch.stack([t[u] for u in units])
    o_ref, S_ref = oracle.prefill_sequential(
        to_np(sel(x["q"])), to_np(sel(x["k"])), to_np(sel(x["v"])), to_np(sel(x["alpha"])),
        to_np(sel(x["beta"])), S0=None if S0 is None else to_np(sel(S0)), per_key=per_key,
        order=order)
    check("o (sampled units)", sel(o32), o_ref, TOL["bf16"])
    check("S_T (sampled units)", sel(S), S_ref, TOL["bf16"])
    return o_ref, S_ref


@pytest.mark.parametrize("name,nunits", [("gdn_prefill", 6), ("long_gdn", 4), ("kda_prefill", 4)])
def test_full_size_prefill(name, nunits):
    w = inputs.workload(name)
    x = inputs.make_inputs(w, seed=0, device="cuda")
    per_key = w.gate == "per_key"
    o32, S = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], per_key=per_key, out="f32")
    o16, S16 = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], per_key=per_key)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    assert o16.dtype == torch.bfloat16 and torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S16, S)
    assert torch.isfinite(o32).all() and torch.isfinite(S).all()
    _check_sampled(x, o32, S, _units(w, nunits, seed=1), per_key)


def test_full_size_prefill_decay_first():
    # the per-key workload in the other order of the per-key factors (bench --order decay_first)
    w = inputs.workload("kda_prefill")
    x = inputs.make_inputs(w, seed=0, device="cuda")
    o32, S = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], per_key=True, out="f32",
                         order="decay_first")
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    assert torch.isfinite(o32).all() and torch.isfinite(S).all()
    _check_sampled(x, o32, S, _units(w, 4, seed=4), True, order="decay_first")


def test_full_size_long_overwrite_invariant():
    # Long-context workload with q_t := k_t at the alpha = beta = 1 positions: the readout
    # there equals v_t up to the deviation of |k_t| from 1 (k is unit-norm before its bf16
    # rounding): |S_t^T k_t - v_t| = |1 - |k_t|^2| |S_{t-1}^T k_t - v_t|.
    w = inputs.workload("long_gdn")
    x = inputs.make_inputs(w, seed=2, device="cuda", q_equals_k_on_subset=True)
    o32, S = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], per_key=False, out="f32")
    torch.cuda.synchronize()
    m = x["subset"][:, :, None, :].expand(w.T, w.B, w.H, w.L)
    v = x["v"][m].float()
    k = x["k"][m].float()
    resid = (o32[m] - v).abs().max(dim=-1).values
    slack = (1 - (k * k).sum(-1)).abs()
    rms = x["v"].float().pow(2).mean().sqrt()
    # the bound with a generous allowance for |S_{t-1}^T k_t - v_t| (a few rms) and the
    # kernel's own error budget
    assert (resid <= TOL["bf16"] * rms + 20 * slack * rms).all()
    units = _units(w, 3, seed=3)
    _check_sampled(x, o32, S, units, False)


def test_full_size_decode():
    # State from a 4096-token prefill of the decode batch, then one decode token per
    # (loop, batch, head); the oracle redoes prefill + step for sampled units from the inputs.
    w = inputs.workload("decode")
    hist = inputs.decode_history(w, seed=0, device="cuda")
    S = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device="cuda")
    lt2.prefill(hist["q"], hist["k"], hist["v"], hist["alpha"], hist["beta"], per_key=False,
                S_out=S, out="f32")
    step = inputs.make_decode_step(w, seed=0, step=0, device="cuda")
    S_dec = S.clone()
    o = lt2.decode(step["q"], step["k"], step["v"], step["alpha"], step["beta"], S_dec,
                   per_key=False, out="f32")
    S_b = S.clone()
    o_b = lt2.decode(step["q"], step["k"], step["v"], step["alpha"], step["beta"], S_b,
                     per_key=False, out="bf16")
    torch.cuda.synchronize()
    assert torch.equal(o_b, o.to(torch.bfloat16)) and torch.equal(S_b, S_dec)
    units = _units(w, 32, seed=4)                # a fixed sample of 32 head-units
    sel = lambda t: torch.stack([t[u] for u in units])
    _, S_hist = oracle.prefill_sequential(to_np(sel(hist["q"])), to_np(sel(hist["k"])),
                                          to_np(sel(hist["v"])), to_np(sel(hist["alpha"])),
                                          to_np(sel(hist["beta"])))
    check("prefilled state (sampled units)", sel(S), S_hist, TOL["bf16"])
    o_ref, S_ref = oracle.decode_step(to_np(sel(step["q"])), to_np(sel(step["k"])),
                                      to_np(sel(step["v"])), to_np(sel(step["alpha"])),
                                      to_np(sel(step["beta"])), S_hist)
    check("decode o (sampled units)", sel(o), o_ref, TOL["bf16"])
    check("decode S (sampled units)", sel(S_dec), S_ref, TOL["bf16"])


@pytest.mark.gpu
def test_prefill_host_equals_device_prefill():
    # inputs in pinned host memory, loops streamed through two device slots with the copies
    # overlapped: the same numbers as the device call, bit for bit
    w = inputs.workload("gdn_prefill", T=3, B=1, H=2, L=200, s0="normal")
    x = inputs.make_inputs(w, seed=4, device="cuda")
    o_ref, S_ref = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=x["S0"], per_key=False)
    h = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta", "S0")}
    o_h = torch.empty(o_ref.shape, dtype=o_ref.dtype).pin_memory()
    S_h = torch.empty(S_ref.shape, dtype=S_ref.dtype).pin_memory()
    lt2.prefill_host(h["q"], h["k"], h["v"], h["alpha"], h["beta"], o_h, S_h, S0=h["S0"])
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(S_h, S_ref.cpu())
