"""Seeded synthetic inputs for the looped gated delta rule.

This module holds no arithmetic of the method itself: it only draws the tensors q, k, v,
alpha, beta and S0 that both the CUDA library and the CPU oracle consume.  It is the one
piece of code the two share.

Workloads (all synthetic; the pages run no public benchmark for this path):

  tiny_fp32    T=2  B=1   H=2  L=64     d=32   fp32 inputs, scalar alpha ~ U[0.9, 1.0]
  gdn_prefill  T=4  B=4   H=16 L=8192   d=128  bf16 q/k/v, scalar alpha
  kda_prefill  T=4  B=2   H=16 L=16384  d=128  bf16 q/k/v, per-key alpha (a d_k vector)
  decode       T=4  B=256 H=16 L=1      d=128  bf16 q/k/v, state from a 4096-token prefill
  long_gdn     T=8  B=1   H=32 L=65536  d=128  bf16, alpha=beta=1 on 1% of the positions
  swa_prefill  T=4  B=4   H=16 L=8192   d=128  bf16 q/k/v, sliding window w=512 (the other mixer)

Distributions: q, k ~ N(0,1) then L2-normalised per (token, head) in fp32 (then cast);
v ~ N(0,1); beta = sigmoid(N(0,1)); alpha = exp(-softplus(N(0,1)) * 0.1) except tiny_fp32
(U[0.9, 1.0]).  Everything is drawn with a torch.Generator seeded by ``seed`` on the
requested device, per loop slice in the order q, k, v, alpha-noise, beta-noise, subset,
then S0.  CPU and CUDA generators give different (but each deterministic) streams, so a
test draws once and hands the same tensors to both sides.
"""
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    B: int
    H: int
    L: int
    d: int
    dtype: str          # "f32" or "bf16": dtype of q, k, v and o
    gate: str           # "scalar" or "per_key"
    alpha_dist: str     # "uniform_0.9_1" or "exp_softplus"
    overwrite_frac: float = 0.0   # fraction of positions with alpha = beta = 1
    history: int = 0    # decode only: tokens of prefill that build the state
    s0: str = "zeros"   # "zeros" or "normal"

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def units(self):
        return self.T * self.B * self.H


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 2, 1, 2, 64, 32, "f32", "scalar", "uniform_0.9_1"),
    "gdn_prefill": Workload("gdn_prefill", 4, 4, 16, 8192, 128, "bf16", "scalar", "exp_softplus"),
    "kda_prefill": Workload("kda_prefill", 4, 2, 16, 16384, 128, "bf16", "per_key", "exp_softplus"),
    "decode": Workload("decode", 4, 256, 16, 1, 128, "bf16", "scalar", "exp_softplus", history=4096),
    "long_gdn": Workload("long_gdn", 8, 1, 32, 65536, 128, "bf16", "scalar", "exp_softplus",
                         overwrite_frac=0.01),
}


def workload(name, **overrides):
    """The named workload, optionally with some fields replaced (e.g. a smaller L)."""
    return replace(WORKLOADS[name], **overrides) if overrides else WORKLOADS[name]


def _normal(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _unit_rows(x):
    # L2 normalisation of each (token, head) row, in fp32.
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(w, seed=0, device="cpu", q_equals_k_on_subset=False):
    """Draw one batch of prefill inputs for workload ``w`` (a Workload).

    Returns a dict with q, k [T,B,H,L,d] and v [T,B,H,L,d] in w's dtype; alpha [T,B,H,L]
    (scalar) or [T,B,H,L,d] (per-key) and beta [T,B,H,L] in fp32; S0 [T,B,H,d,d] fp32 or
    None; and "subset" (a [T,B,L] bool mask of overwrite positions, or None).
    With ``q_equals_k_on_subset`` the query at an overwrite position is set to its key.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    T, B, H, L, d = w.T, w.B, w.H, w.L, w.d
    dt = w.torch_dtype
    q = torch.empty((T, B, H, L, d), dtype=dt, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    ashape = (T, B, H, L, d) if w.gate == "per_key" else (T, B, H, L)
    alpha = torch.empty(ashape, dtype=torch.float32, device=device)
    beta = torch.empty((T, B, H, L), dtype=torch.float32, device=device)
    subset = None
    if w.overwrite_frac > 0:
        subset = torch.zeros((T, B, L), dtype=torch.bool, device=device)
    for t in range(T):
        qs = _unit_rows(_normal((B, H, L, d), gen, device))
        ks = _unit_rows(_normal((B, H, L, d), gen, device))
        q[t] = qs.to(dt)
        k[t] = ks.to(dt)
        del qs, ks
        v[t] = _normal((B, H, L, d), gen, device).to(dt)
        if w.alpha_dist == "uniform_0.9_1":
            u = torch.rand(ashape[1:], generator=gen, device=device, dtype=torch.float32)
            alpha[t] = 0.9 + 0.1 * u
        else:
            x = _normal(ashape[1:], gen, device)
            alpha[t] = torch.exp(-torch.nn.functional.softplus(x) * 0.1)
        beta[t] = torch.sigmoid(_normal((B, H, L), gen, device))
        if subset is not None:
            n_sel = int(round(w.overwrite_frac * L))
            for b in range(B):
                pos = torch.randperm(L, generator=gen, device=device)[:n_sel]
                subset[t, b, pos] = True
            m = subset[t][:, None, :].expand(B, H, L)
            alpha[t][m] = 1.0          # per-key: the whole d_k vector of the position
            beta[t][m] = 1.0
            if q_equals_k_on_subset:
                q[t][m] = k[t][m]
    S0 = None
    if w.s0 == "normal":
        S0 = _normal((T, B, H, d, d), gen, device)
    return {"q": q, "k": k, "v": v, "alpha": alpha, "beta": beta, "S0": S0, "subset": subset}


def make_decode_step(w, seed=0, step=0, device="cpu"):
    """One decode token per (loop, batch, head): q, k, v [T,B,H,d]; alpha [T,B,H] (or
    [T,B,H,d] per-key); beta [T,B,H].  Drawn like the prefill inputs of ``w``."""
    one = replace(w, L=1, overwrite_frac=0.0, s0="zeros")
    x = make_inputs(one, seed=seed * 1_000_003 + 7919 * (step + 1), device=device)
    out = {n: x[n][..., 0, :] if n in ("q", "k", "v") else x[n][:, :, :, 0]
           for n in ("q", "k", "v", "alpha", "beta")}
    return out


def decode_history(w, seed=0, device="cpu"):
    """The prefill inputs (L = w.history tokens) whose final state seeds the decode."""
    return make_inputs(replace(w, L=w.history, overwrite_frac=0.0), seed=seed, device=device)


def make_raw_inputs(w, seed=0, device="cpu"):
    """The raw projections of the fused prologue and output gate for workload ``w``: q, k and the
    output gate logits z ~ N(0,1) in w's dtype (q and k NOT normalised), and N(0,1) logits a (the
    shape of alpha: [T,B,H,L] or [T,B,H,L,d]) and b ([T,B,H,L]) in fp32; v ~ N(0,1); S0 as in
    make_inputs.  Drawn in the order q, k, v, z, a, b, then S0."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    T, B, H, L, d = w.T, w.B, w.H, w.L, w.d
    dt = w.torch_dtype
    shape = (T, B, H, L, d)
    q = _normal(shape, gen, device).to(dt)
    k = _normal(shape, gen, device).to(dt)
    v = _normal(shape, gen, device).to(dt)
    z = _normal(shape, gen, device).to(dt)
    a = _normal((T, B, H, L, d) if w.gate == "per_key" else (T, B, H, L), gen, device)
    b = _normal((T, B, H, L), gen, device)
    S0 = _normal((T, B, H, d, d), gen, device) if w.s0 == "normal" else None
    return {"q": q, "k": k, "v": v, "z": z, "a": a, "b": b, "S0": S0}


@dataclass(frozen=True)
class SwaWorkload:
    """A sliding-window attention prefill: T loops x B x H units of L tokens, head width d."""
    name: str
    T: int
    B: int
    H: int
    L: int
    d: int
    window: int
    dtype: str = "bf16"

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def units(self):
        return self.T * self.B * self.H


SWA_WORKLOADS = {
    "swa_prefill": SwaWorkload("swa_prefill", 4, 4, 16, 8192, 128, 512),
}


def swa_workload(name, **overrides):
    return replace(SWA_WORKLOADS[name], **overrides) if overrides else SWA_WORKLOADS[name]


def make_swa_inputs(w, seed=0, device="cpu"):
    """q, k, v ~ N(0,1) [T,B,H,L,d] in w's dtype (drawn in fp32 in that order, then cast): with
    the default scale 1/sqrt(d) the scores q.k/sqrt(d) are ~N(0,1)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    shape = (w.T, w.B, w.H, w.L, w.d)
    q = _normal(shape, gen, device).to(w.torch_dtype)
    k = _normal(shape, gen, device).to(w.torch_dtype)
    v = _normal(shape, gen, device).to(w.torch_dtype)
    return {"q": q, "k": k, "v": v}
