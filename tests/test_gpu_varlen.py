"""Packed sequences of different lengths (lt2_gdr_prefill_varlen) on every path, against the
fp64 packed-sequence oracle of oracle/varlen.py on the same inputs.

Each (loop, sequence, head) is its own recurrence ("LT2 transformer looped a tempo lineare",
section "Sostituire il motore", displayed equation); sequence b owns tokens cu[b] .. cu[b+1]-1
of every (loop, head).  Lengths mix a single token, one chunk exactly, chunk +- 1, several chunks
with a ragged tail and an empty sequence, so the tensor-core kernel's masked last chunk (whose
rows past the end belong to the next sequence) is exercised at every position.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import inputs
from oracle import varlen as ovarlen
from tests.gpu_util import TOL, check, to_np

pytestmark = pytest.mark.gpu

TC, CC = lt2.LT2_ALGO_TENSOR_CORE, lt2.LT2_ALGO_CUDA_CORE
LENS = [1, 63, 64, 65, 200, 0, 130, 7]


def _x(lens, seed, T=2, H=2, d=128, dtype="bf16", gate="scalar"):
    N = int(sum(lens))
    w = inputs.workload("kda_prefill" if gate == "per_key" else "gdn_prefill", T=T, B=1, H=H, L=N, d=d,
                        dtype=dtype, s0="normal")
    x = inputs.make_inputs(w, seed=seed, device="cuda")
    out = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "alpha", "beta")}   # [T, H, N, ...]
    B = len(lens)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    out["S0"] = torch.randn((T, B, H, d, d), generator=g, device="cuda")
    out["cu"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device="cuda")
    return out


def _run(x, algo=lt2.LT2_ALGO_AUTO, out="f32", per_key=False, order="delta_first", **kw):
    o, S = lt2.prefill_varlen(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["cu"], S0=x["S0"], algo=algo,
                              out=out, per_key=per_key, order=order, **kw)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
    return o, S


def _ref(x, per_key=False, order="delta_first"):
    return ovarlen.prefill(*(to_np(x[n]) for n in ("q", "k", "v", "alpha", "beta")), to_np(x["cu"]),
                           S0=to_np(x["S0"]), per_key=per_key, order=order)


@pytest.mark.parametrize("algo", [TC, CC])
def test_scalar_bf16_matches_oracle(algo):
    x = _x(LENS, seed=1)
    o, S = _run(x, algo)
    o_ref, S_ref = _ref(x)
    check("o (varlen)", o, o_ref, TOL["bf16"])
    check("S_T (varlen)", S, S_ref, TOL["bf16"])


def test_tensor_core_bf16_output_is_rounded_fp32_output():
    x = _x(LENS, seed=2)
    o32, S32 = _run(x, TC, out="f32")
    o16, S16 = _run(x, TC, out="bf16")
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S32)


def test_tensor_core_equal_lengths_equal_the_fixed_layout():
    # B sequences of one length through the packed call give the fixed-layout call's numbers
    T, B, H, L = 2, 3, 2, 150
    x = _x([L] * B, seed=3, T=T, H=H)
    o, S = _run(x, TC, out="bf16")
    unpack = lambda t: t.reshape(T, H, B, L, *t.shape[3:]).transpose(1, 2).contiguous()
    of, Sf = lt2.prefill(unpack(x["q"]), unpack(x["k"]), unpack(x["v"]), unpack(x["alpha"]), unpack(x["beta"]),
                         S0=x["S0"], per_key=False, algo=TC, out="bf16")
    torch.cuda.synchronize()
    assert torch.equal(unpack(o), of) and torch.equal(S, Sf)


def test_tensor_core_leaves_rows_outside_the_sequences_alone():
    # a sequence's masked last chunk writes only that sequence's rows: a sentinel in the rows that
    # no sequence covers survives, with fp32 output (plain stores) and with bf16 output (box
    # stores for whole chunks, 16-byte stores for the last one); the covered rows match the oracle
    lens = [70, 0, 3]
    x = _x(lens + [40], seed=4)
    x["cu"] = x["cu"][:-1].contiguous()                      # the last 40 rows belong to no sequence
    x["S0"] = x["S0"][:, :3].contiguous()
    outs = {}
    for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        o = torch.full(x["v"].shape, 7.0, dtype=dt, device="cuda")
        lt2.prefill_varlen(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["cu"], S0=x["S0"], algo=TC, o=o, out=name)
        torch.cuda.synchronize()
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        assert torch.all(o[:, :, 73:] == 7.0)
        outs[name] = o
    o_ref, _ = _ref(x)
    check("o (sequences)", outs["f32"][:, :, :73], o_ref[:, :, :73], TOL["bf16"])
    assert torch.equal(outs["bf16"][:, :, :73], outs["f32"][:, :, :73].to(torch.bfloat16))


# the per-key kernel works in 32-token chunks: lengths around one and several of them
LENS_PK = [1, 31, 32, 33, 100, 0, 70, 7]
ORDERS = ["delta_first", "decay_first"]


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("algo", [TC, CC])
def test_per_key_bf16_matches_oracle(algo, order):
    x = _x(LENS_PK, seed=5, gate="per_key")
    o, S = _run(x, algo, per_key=True, order=order)
    o_ref, S_ref = _ref(x, per_key=True, order=order)
    check("o (per-key varlen)", o, o_ref, TOL["bf16"])
    check("S_T (per-key varlen)", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("order", ORDERS)
def test_per_key_tensor_core_bf16_output_is_rounded_fp32_output(order):
    x = _x(LENS_PK, seed=9, gate="per_key")
    o32, S32 = _run(x, TC, out="f32", per_key=True, order=order)
    o16, S16 = _run(x, TC, out="bf16", per_key=True, order=order)
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S32)


@pytest.mark.parametrize("order", ORDERS)
def test_per_key_tensor_core_equal_lengths_equal_the_fixed_layout(order):
    # B sequences of one length (4 chunks and a ragged 22-token tail) through the packed call give
    # the fixed-layout call's numbers
    T, B, H, L = 2, 3, 2, 150
    x = _x([L] * B, seed=10, T=T, H=H, gate="per_key")
    o, S = _run(x, TC, out="bf16", per_key=True, order=order)
    unpack = lambda t: t.reshape(T, H, B, L, *t.shape[3:]).transpose(1, 2).contiguous()
    of, Sf = lt2.prefill(unpack(x["q"]), unpack(x["k"]), unpack(x["v"]), unpack(x["alpha"]), unpack(x["beta"]),
                         S0=x["S0"], per_key=True, algo=TC, out="bf16", order=order)
    torch.cuda.synchronize()
    assert torch.equal(unpack(o), of) and torch.equal(S, Sf)


@pytest.mark.parametrize("order", ORDERS)
def test_per_key_tensor_core_exact_chunks_on_packed_sequences(order):
    # alpha^6 puts most chunks beyond the fp16 tile range (run token by token inside the kernel)
    # and a zeroed alpha row is a reset: the packed instances' exact path, at every position of a
    # sequence (first chunk, middle, a partial last chunk)
    x = _x([100, 33, 0, 64, 7], seed=13, gate="per_key")
    x["alpha"] = x["alpha"].double().pow(6.0).float()
    x["alpha"][:, :, 40, :] = 0.0
    x["alpha"][:, :, 120, 3] = 0.0
    o, S = _run(x, TC, per_key=True, order=order)
    o_ref, S_ref = _ref(x, per_key=True, order=order)
    check("o (per-key varlen, exact chunks)", o, o_ref, TOL["bf16"])
    check("S_T (per-key varlen, exact chunks)", S, S_ref, TOL["bf16"])


def test_per_key_tensor_core_leaves_rows_outside_the_sequences_alone():
    lens = [40, 0, 3]
    x = _x(lens + [30], seed=11, gate="per_key")
    x["cu"] = x["cu"][:-1].contiguous()                      # the last 30 rows belong to no sequence
    x["S0"] = x["S0"][:, :3].contiguous()
    outs = {}
    for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        o = torch.full(x["v"].shape, 7.0, dtype=dt, device="cuda")
        lt2.prefill_varlen(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["cu"], S0=x["S0"], algo=TC, o=o,
                           out=name, per_key=True)
        torch.cuda.synchronize()
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        assert torch.all(o[:, :, 43:] == 7.0)
        outs[name] = o
    o_ref, _ = _ref(x, per_key=True)
    check("o (per-key sequences)", outs["f32"][:, :, :43], o_ref[:, :, :43], TOL["bf16"])
    assert torch.equal(outs["bf16"][:, :, :43], outs["f32"][:, :, :43].to(torch.bfloat16))


def test_per_key_fused_steps_on_packed_sequences():
    lens = [50, 1, 32, 29]
    N, T, H = sum(lens), 2, 2
    w = inputs.workload("kda_prefill", T=T, B=1, H=H, L=N)
    r = inputs.make_raw_inputs(w, seed=12, device="cuda")
    x = {n: r[n][:, 0].contiguous() for n in ("q", "k", "v", "z", "a", "b")}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device="cuda")
    for algo in (TC, CC):
        o, S = lt2.prefill_varlen(x["q"], x["k"], x["v"], x["a"], x["b"], cu, algo=algo, out="f32", per_key=True,
                                  qk_l2norm=True, gate_logits=True, alpha_scale=0.1, z=x["z"])
        torch.cuda.synchronize()
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        o_ref, S_ref = ovarlen.prefill(*(to_np(x[n]) for n in ("q", "k", "v", "a", "b")), to_np(cu), per_key=True,
                                       raw=dict(z=to_np(x["z"]), alpha_scale=0.1))
        check(f"o (per-key fused varlen, algo {algo})", o, o_ref, TOL["bf16"])
        check(f"S_T (per-key fused varlen, algo {algo})", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_fp32_cuda_core_is_exact(gate):
    x = _x([9, 1, 40, 0, 17], seed=6, d=32, dtype="f32", gate=gate)
    o, S = _run(x, per_key=gate == "per_key")
    o_ref, S_ref = _ref(x, per_key=gate == "per_key")
    check("o (fp32 varlen)", o, o_ref, TOL["f32"])
    check("S_T (fp32 varlen)", S, S_ref, TOL["f32"])


def test_fused_steps_on_packed_sequences():
    lens = [100, 1, 64, 29]
    N, T, H = sum(lens), 2, 2
    w = inputs.workload("gdn_prefill", T=T, B=1, H=H, L=N)
    r = inputs.make_raw_inputs(w, seed=7, device="cuda")
    x = {n: r[n][:, 0].contiguous() for n in ("q", "k", "v", "z", "a", "b")}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device="cuda")
    for algo in (TC, CC):
        o, S = lt2.prefill_varlen(x["q"], x["k"], x["v"], x["a"], x["b"], cu, algo=algo, out="f32", qk_l2norm=True,
                                  gate_logits=True, alpha_scale=0.1, z=x["z"])
        torch.cuda.synchronize()
        assert lt2.lt2_gdr_last_device_error() == lt2.LT2_OK
        o_ref, S_ref = ovarlen.prefill(*(to_np(x[n]) for n in ("q", "k", "v", "a", "b")), to_np(cu),
                                       raw=dict(z=to_np(x["z"]), alpha_scale=0.1))
        check(f"o (fused varlen, algo {algo})", o, o_ref, TOL["bf16"])
        check(f"S_T (fused varlen, algo {algo})", S, S_ref, TOL["bf16"])


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("algo", [TC, CC])
def test_bad_offsets_are_reported(algo, gate):
    pk = gate == "per_key"
    x = _x([10, 20, 30], seed=8, gate=gate)
    x["cu"] = torch.tensor([0, 20, 10, 60], dtype=torch.int64, device="cuda")     # out of order
    lt2.prefill_varlen(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["cu"], S0=x["S0"], algo=algo, per_key=pk)
    torch.cuda.synchronize()
    assert lt2.lt2_gdr_last_device_error() == lt2.LT2_ERR_SEQLENS
    # and the context is fine afterwards
    x["cu"] = torch.tensor([0, 10, 30, 60], dtype=torch.int64, device="cuda")
    o, S = _run(x, algo, per_key=pk)
    o_ref, S_ref = _ref(x, per_key=pk)
    check("o (after bad offsets)", o, o_ref, TOL["bf16"])
