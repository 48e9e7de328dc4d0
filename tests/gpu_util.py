"""Helpers for the GPU parity tests: run the library and the oracle on the same inputs."""
import numpy as np
import torch

import gated_delta_rule_looped_b200 as lt2
import oracle

TOL = {"f32": 1e-4, "bf16": 2e-2}   # max|gpu - ref| / rms(ref), per output tensor

# Parity is checked on an fp32 copy of o: the final rounding of o to bf16 alone can reach
# 2^-8 |o|, i.e. ~2e-2 of rms(o) at the largest |o| of a big tensor, whatever the kernel
# does.  The bf16 output is checked separately to be exactly the fp32 output rounded to
# nearest-even.


def to_np(x):
    return None if x is None else x.detach().to("cpu", torch.float64).numpy()


def oracle_prefill(x, per_key, units=None, order="delta_first"):
    """fp64 oracle on (a subset of) the head-units of input dict x.  ``units`` is a list of
    (tau, b, h) triples, or None for all."""
    sel = (lambda t: t) if units is None else (lambda t: torch.stack([t[u] for u in units]))
    S0 = None if x.get("S0") is None else to_np(sel(x["S0"]))
    return oracle.prefill_sequential(to_np(sel(x["q"])), to_np(sel(x["k"])), to_np(sel(x["v"])),
                                     to_np(sel(x["alpha"])), to_np(sel(x["beta"])), S0=S0,
                                     per_key=per_key, order=order)


def check(name, got, ref, tol):
    err = oracle.rel_max_err(to_np(got) if isinstance(got, torch.Tensor) else got, ref)
    assert np.isfinite(err) and err <= tol, f"{name}: rel max err {err:.3e} > {tol:.1e}"
    return err


def to_device(x, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_prefill(x, per_key, algo=lt2.LT2_ALGO_AUTO, S0=None, out="f32", order="delta_first"):
    o, S = lt2.prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                       S0=x.get("S0") if S0 is None else S0, per_key=per_key, algo=algo,
                       out=out, order=order)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    return o, S
