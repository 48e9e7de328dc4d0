"""The C-ABI library on the CPU: it loads, exports every symbol include/lt2_gdr.h declares,
and rejects bad arguments synchronously with the documented status, before touching the GPU
(every call below fails validation, so nothing is launched; pointers are fake addresses).
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_looped_b200 as lt2
from gated_delta_rule_looped_b200 import build as lbuild

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module")
def L():
    if lbuild.needs_build():
        lbuild.build()
    return lt2.lib()


def _declared_functions(header="lt2_gdr.h"):
    with open(os.path.join(HEADER_DIR, header)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(lt2_\w+)\s*\(", text))


def test_headers_are_the_product_and_the_debug_header():
    assert sorted(f for f in os.listdir(HEADER_DIR) if f.endswith(".h")) == ["lt2_gdr.h", "lt2_gdr_debug.h"]


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert declared, "no declarations found"
    assert declared == set(lt2.EXPORTS)
    for name in declared:
        assert hasattr(L, name), f"{name} not exported"


def test_debug_library_exports_both_headers_and_product_only_its_own():
    if lbuild.needs_build(debug=True):
        lbuild.build(debug=True)
    D = ctypes.CDLL(lbuild.DEBUG_LIB)
    debug_only = _declared_functions("lt2_gdr_debug.h")
    assert debug_only == {"lt2_debug_set_skip_chunk", "lt2_debug_wait_timeout_ns"}
    for name in _declared_functions() | debug_only:
        assert hasattr(D, name), f"{name} not exported by the debug library"
    P = ctypes.CDLL(lbuild.LIB)
    for name in debug_only:
        assert not hasattr(P, name), f"the product library exports the test hook {name}"
    D.lt2_debug_wait_timeout_ns.restype = ctypes.c_uint64
    assert 0 < D.lt2_debug_wait_timeout_ns() <= 100_000_000     # milliseconds, not seconds


def test_status_strings(L):
    for code, name in [(0, "LT2_OK"), (1, "LT2_ERR_INVALID_ARGUMENT"), (2, "LT2_ERR_UNSUPPORTED"),
                       (3, "LT2_ERR_WORKSPACE"), (4, "LT2_ERR_CUDA"),
                       (5, "LT2_ERR_DEVICE_TIMEOUT"), (6, "LT2_ERR_RANGE"),
                       (7, "LT2_ERR_DEVICE_CHECK")]:
        assert lt2.lt2_status_string(code) == name
    assert lt2.lt2_status_string(99) == "LT2_STATUS_UNKNOWN"
    assert L.lt2_gdr_version() >= 200


def test_dims_struct_layout():
    assert ctypes.sizeof(lt2.lt2_gdr_dims) == 6 * 8 + 4 * 4


# Fake, 16-byte aligned, non-overlapping "device" addresses (never dereferenced).
BASE = 1 << 40
SPAN = 1 << 34


def addrs(n):
    return [BASE + i * SPAN for i in range(n)]


def call_prefill(dims, **over):
    q, k, v, a, b, s0, o, so = addrs(8)
    args = dict(q=q, k=k, v=v, alpha=a, beta=b, S0=s0, o=o, S_out=so)
    args.update(over)
    return lt2.lt2_gdr_prefill(dims, args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                               args["S0"], args["o"], args["S_out"], None, 0, 0)


def call_decode(dims, **over):
    q, k, v, a, b, S, o = addrs(7)
    args = dict(q=q, k=k, v=v, alpha=a, beta=b, S=S, o=o)
    args.update(over)
    return lt2.lt2_gdr_decode(dims, args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                              args["S"], args["o"], 0)


def D(**kw):
    base = dict(T=2, B=1, H=2, L=64, dk=32, dv=32, dtype=lt2.LT2_DTYPE_F32,
                gate=lt2.LT2_GATE_SCALAR, algo=lt2.LT2_ALGO_AUTO)
    base.update(kw)
    return lt2.make_dims(**base)


def test_null_dims_rejected(L):
    st = L.lt2_gdr_prefill(None, 1, 1, 1, 1, 1, None, 1, None, None, 0, None)
    assert st == lt2.LT2_ERR_INVALID_ARGUMENT
    assert L.lt2_gdr_prefill_workspace_bytes(None) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(dk=256, dv=256), lt2.LT2_ERR_UNSUPPORTED),
    (dict(dk=12), lt2.LT2_ERR_UNSUPPORTED),
    (dict(dv=130), lt2.LT2_ERR_UNSUPPORTED),
    (dict(dk=0), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(L=-1), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(T=-2), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(dtype=7), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(gate=3), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(algo=9), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(algo=lt2.LT2_ALGO_TENSOR_CORE), lt2.LT2_ERR_UNSUPPORTED),   # fp32, d=32
    (dict(T=1 << 30, B=1 << 30, H=1 << 30), lt2.LT2_ERR_INVALID_ARGUMENT),
])
def test_bad_dims(L, kw, status):
    assert call_prefill(D(**kw)) == status


def test_bad_out_dtype(L):
    d = D()
    d.out_dtype = 3
    assert call_prefill(d) == lt2.LT2_ERR_INVALID_ARGUMENT
    d.out_dtype = -1
    assert call_prefill(d) == lt2.LT2_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field", ["q", "k", "v", "alpha", "beta", "o"])
def test_null_pointer_rejected(L, field):
    assert call_prefill(D(), **{field: None}) == lt2.LT2_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field", ["q", "k", "v", "alpha", "beta", "o", "S0", "S_out"])
def test_misaligned_pointer_rejected(L, field):
    assert call_prefill(D(), **{field: BASE + 20 * SPAN + 8}) == lt2.LT2_ERR_INVALID_ARGUMENT


def test_aliasing_rejected(L):
    q = addrs(1)[0]
    assert call_prefill(D(), o=q + 64) == lt2.LT2_ERR_INVALID_ARGUMENT        # o inside q
    s0 = addrs(6)[5]
    assert call_prefill(D(), S_out=s0 + 256) == lt2.LT2_ERR_INVALID_ARGUMENT  # partial overlap
    o = addrs(7)[6]
    assert call_prefill(D(), S_out=o) == lt2.LT2_ERR_INVALID_ARGUMENT


def test_empty_problem_is_a_noop(L):
    # No head-units: valid, nothing to launch, no GPU needed.
    assert call_prefill(D(T=0)) == lt2.LT2_OK
    assert call_prefill(D(B=0), q=None, k=None, v=None, alpha=None, beta=None, o=None) == lt2.LT2_OK


def test_workspace_query(L):
    assert lt2.lt2_gdr_prefill_workspace_bytes(D()) == 0
    assert lt2.lt2_gdr_prefill_workspace_bytes(D(dk=7)) == 0


def test_decode_validation(L):
    assert call_decode(D(L=64)) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_decode(D(L=1), S=None) == lt2.LT2_ERR_INVALID_ARGUMENT
    S = addrs(7)[5]
    assert call_decode(D(L=1), o=S) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_decode(D(L=1, dk=136)) == lt2.LT2_ERR_UNSUPPORTED
    assert call_decode(D(L=1, B=0)) == lt2.LT2_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(lt2, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(lt2, "_LIB", None)
    with pytest.raises(ImportError):
        lt2.lib()


@pytest.mark.parametrize("gate", [lt2.LT2_GATE_PER_KEY, lt2.LT2_GATE_PER_KEY_DECAY_FIRST])
def test_per_key_gates_take_per_key_alpha(L, gate):
    # alpha of either per-key gate holds T*B*H*L*dk floats: an o placed past the scalar extent
    # (T*B*H*L floats) but inside the per-key one overlaps it
    a = addrs(4)[3]
    tok = 2 * 1 * 2 * 64
    assert call_prefill(D(gate=gate), o=a + tok * 4 + 64) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_prefill(D(gate=gate, T=0)) == lt2.LT2_OK


def test_order_names_checked():
    assert lt2._gate(True, "decay_first") == lt2.LT2_GATE_PER_KEY_DECAY_FIRST
    assert lt2._gate(True, "delta_first") == lt2.LT2_GATE_PER_KEY
    assert lt2._gate(False, "decay_first") == lt2.LT2_GATE_SCALAR
    with pytest.raises(ValueError):
        lt2._gate(True, "decay_last")


def test_binding_rejects_tensors_it_cannot_pass_by_pointer():
    # the convenience layer checks device, contiguity, shape and dtype before calling the ABI
    import torch
    q = torch.zeros((1, 1, 1, 4, 128), dtype=torch.bfloat16)
    a = torch.ones((1, 1, 1, 4), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        lt2.prefill(q, q, q, a, a)
    with pytest.raises(ValueError, match="CUDA"):
        lt2.decode(q[..., 0, :], q[..., 0, :], q[..., 0, :], a[..., 0], a[..., 0],
                   torch.zeros((1, 1, 1, 128, 128)))


# ---- the fused entry points: their descriptor is validated before any launch ----------------

def call_prefill_fused(dims, fused, **over):
    q, k, v, a, b, s0, o, so = addrs(8)
    args = dict(q=q, k=k, v=v, alpha=a, beta=b, S0=s0, o=o, S_out=so)
    args.update(over)
    return lt2.lt2_gdr_prefill_fused(dims, fused, args["q"], args["k"], args["v"], args["alpha"],
                                     args["beta"], args["S0"], args["o"], args["S_out"], None, 0, 0)


def test_fused_descriptor_layout():
    assert ctypes.sizeof(lt2.lt2_gdr_fused) == 24
    assert lt2.lt2_gdr_fused.z.offset == 16


@pytest.mark.parametrize("field,value", [("reserved", 1), ("qk_l2norm", 2), ("gate_logits", -1)])
def test_fused_bad_fields_rejected(L, field, value):
    f = lt2.make_fused(True, True, 0.1)
    setattr(f, field, value)
    assert call_prefill_fused(D(), f) == lt2.LT2_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("scale", [-0.5, float("nan"), float("inf")])
def test_fused_bad_alpha_scale_rejected(L, scale):
    assert call_prefill_fused(D(), lt2.make_fused(False, True, scale)) == lt2.LT2_ERR_INVALID_ARGUMENT


def test_fused_z_checked(L):
    q, k, v, a, b, s0, o, so = addrs(8)
    assert call_prefill_fused(D(), lt2.make_fused(z=o + 64)) == lt2.LT2_ERR_INVALID_ARGUMENT     # overlaps o
    assert call_prefill_fused(D(), lt2.make_fused(z=BASE + 9 * SPAN + 4)) == lt2.LT2_ERR_INVALID_ARGUMENT  # misaligned
    dims = D(L=1)
    assert lt2.lt2_gdr_decode_fused(dims, lt2.make_fused(z=o), q, k, v, a, b, s0, o, 0) == \
        lt2.LT2_ERR_INVALID_ARGUMENT


def test_fused_null_descriptor_is_the_plain_call(L):
    # validation runs the same way: a bad dims fails identically with and without a descriptor
    bad = D(dk=0)
    assert call_prefill_fused(bad, None) == call_prefill(bad) == lt2.LT2_ERR_INVALID_ARGUMENT


# ---- the sliding-window mixer (lt2_swa_prefill) ------------------------------------------------

def SD(**kw):
    base = dict(T=2, B=1, H=2, L=64, d=32, window=8, scale=0.0, dtype=lt2.LT2_DTYPE_F32,
                algo=lt2.LT2_ALGO_AUTO, out_dtype=lt2.LT2_OUT_SAME)
    base.update(kw)
    return lt2.lt2_swa_dims(**base)


def call_swa(dims, **over):
    q, k, v, o = addrs(4)
    args = dict(q=q, k=k, v=v, o=o)
    args.update(over)
    return lt2.lt2_swa_prefill(dims, args["q"], args["k"], args["v"], args["o"], 0)


def test_swa_dims_struct_layout():
    assert ctypes.sizeof(lt2.lt2_swa_dims) == 6 * 8 + 4 * 4
    assert lt2.lt2_swa_dims.scale.offset == 48


@pytest.mark.parametrize("kw,status", [
    (dict(window=0), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(window=-3), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(d=0), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(L=-1), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(scale=-1.0), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(scale=float("inf")), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(dtype=5), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(algo=7), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(out_dtype=3), lt2.LT2_ERR_INVALID_ARGUMENT),
    (dict(d=257), lt2.LT2_ERR_UNSUPPORTED),
    (dict(algo=lt2.LT2_ALGO_TENSOR_CORE), lt2.LT2_ERR_UNSUPPORTED),                           # fp32
    (dict(algo=lt2.LT2_ALGO_TENSOR_CORE, dtype=lt2.LT2_DTYPE_BF16, d=64), lt2.LT2_ERR_UNSUPPORTED),
    (dict(T=1 << 30, B=1 << 30, H=1 << 30), lt2.LT2_ERR_INVALID_ARGUMENT),
])
def test_swa_bad_dims(L, kw, status):
    assert call_swa(SD(**kw)) == status


def test_swa_null_dims_rejected(L):
    assert L.lt2_swa_prefill(None, 1 << 40, 1 << 40, 1 << 40, 1 << 41, None) == lt2.LT2_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field", ["q", "k", "v", "o"])
def test_swa_null_or_misaligned_pointer_rejected(L, field):
    assert call_swa(SD(), **{field: None}) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_swa(SD(), **{field: BASE + 20 * SPAN + 8}) == lt2.LT2_ERR_INVALID_ARGUMENT


def test_swa_aliasing_rejected(L):
    q, k, v, o = addrs(4)
    assert call_swa(SD(), o=q) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_swa(SD(), o=v + 256) == lt2.LT2_ERR_INVALID_ARGUMENT


def test_swa_empty_problem_is_a_noop(L):
    assert call_swa(SD(T=0)) == lt2.LT2_OK
    assert call_swa(SD(L=0), q=None, k=None, v=None, o=None) == lt2.LT2_OK


# ---- packed sequences (lt2_gdr_prefill_varlen) ---------------------------------------------

def call_varlen(dims, cu=BASE + 30 * SPAN, **over):
    q, k, v, a, b, s0, o, so = addrs(8)
    args = dict(q=q, k=k, v=v, alpha=a, beta=b, S0=s0, o=o, S_out=so)
    args.update(over)
    return lt2.lt2_gdr_prefill_varlen(dims, None, cu, args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                                      args["S0"], args["o"], args["S_out"], None, 0, 0)


def test_varlen_offsets_checked(L):
    assert call_varlen(D(), cu=None) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_varlen(D(), cu=BASE + 30 * SPAN + 4) == lt2.LT2_ERR_INVALID_ARGUMENT     # not 8-byte aligned
    q = addrs(1)[0]
    assert call_varlen(D(), o=q + 64) == lt2.LT2_ERR_INVALID_ARGUMENT                    # o inside q
    assert call_varlen(D(), cu=addrs(7)[6] + 16) == lt2.LT2_ERR_INVALID_ARGUMENT        # offsets inside o


def test_varlen_tensor_core_needs_bf16_and_d128(L):
    # both gatings have a tensor-core varlen path for bf16 inputs at d = 128, and only there
    for gate in (lt2.LT2_GATE_SCALAR, lt2.LT2_GATE_PER_KEY, lt2.LT2_GATE_PER_KEY_DECAY_FIRST):
        for over in (dict(dtype=lt2.LT2_DTYPE_F32, dk=128, dv=128), dict(dtype=lt2.LT2_DTYPE_BF16, dk=64, dv=64)):
            d = D(gate=gate, algo=lt2.LT2_ALGO_TENSOR_CORE, **over)
            assert call_varlen(d) == lt2.LT2_ERR_UNSUPPORTED


def test_varlen_bad_dims_and_empty(L):
    assert call_varlen(D(dk=0)) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_varlen(D(T=0)) == lt2.LT2_OK
    assert L.lt2_gdr_prefill_varlen(None, None, BASE, 1, 1, 1, 1, 1, None, 1, None, None, 0, None) == \
        lt2.LT2_ERR_INVALID_ARGUMENT


def test_seqlens_status_has_a_name(L):
    assert lt2.lt2_status_string(lt2.LT2_ERR_SEQLENS) == "LT2_ERR_SEQLENS"


# ---- backward (lt2_gdr_backward) ------------------------------------------------------------

def call_backward(dims, ws=BASE + 40 * SPAN, ws_bytes=None, **over):
    a = addrs(16)
    names = ["q", "k", "v", "alpha", "beta", "S0", "dO", "dS_L", "dq", "dk", "dv", "dalpha", "dbeta", "dS0"]
    args = dict(zip(names, a))
    args.update(over)
    if ws_bytes is None:
        ws_bytes = lt2.lt2_gdr_backward_workspace_bytes(dims)
    return lt2.lt2_gdr_backward(dims, *(args[n] for n in names), ws, ws_bytes, 0)


def test_prefill_workspace_query(L):
    # one 4-byte flag per unit, rounded up to 256 bytes, for the scalar bf16 d = 128 tensor-core
    # prefill (its balanced schedule); 0 for the per-key kernel and the CUDA-core path
    d = D(dtype=lt2.LT2_DTYPE_BF16, dk=128, dv=128, T=3, B=2, H=50)
    assert lt2.lt2_gdr_prefill_workspace_bytes(d) == (3 * 2 * 50 * 4 + 255) // 256 * 256
    assert lt2.lt2_gdr_prefill_workspace_bytes(D(dtype=lt2.LT2_DTYPE_BF16, dk=128, dv=128,
                                                gate=lt2.LT2_GATE_PER_KEY)) == 0
    assert lt2.lt2_gdr_prefill_workspace_bytes(D(dtype=lt2.LT2_DTYPE_BF16, dk=128, dv=128,
                                                algo=lt2.LT2_ALGO_CUDA_CORE)) == 0
    assert lt2.lt2_gdr_prefill_workspace_bytes(D()) == 0                   # fp32, d = 32


def test_backward_workspace_query(L):
    d = D(L=150)
    units, chunks, slices = 2 * 1 * 2, 5, 1                      # d = 32: one 32-column slice
    # a checkpoint every 32 tokens (ceil(150 / 32) = 5) and the 33 states of one chunk, d_k x 32 fp32 each
    assert lt2.lt2_gdr_backward_workspace_bytes(d) == units * slices * (chunks + 33) * 32 * 32 * 4
    assert L.lt2_gdr_backward_workspace_bytes(None) == 0


def test_backward_validation(L):
    assert call_backward(D(dk=0)) == lt2.LT2_ERR_INVALID_ARGUMENT
    assert call_backward(D(algo=lt2.LT2_ALGO_TENSOR_CORE)) == lt2.LT2_ERR_UNSUPPORTED
    assert call_backward(D(), ws=None) == lt2.LT2_ERR_WORKSPACE
    assert call_backward(D(), ws_bytes=16) == lt2.LT2_ERR_WORKSPACE
    assert call_backward(D(), dq=None) == lt2.LT2_ERR_INVALID_ARGUMENT
    q = addrs(1)[0]
    assert call_backward(D(), dq=q) == lt2.LT2_ERR_INVALID_ARGUMENT          # a gradient over an input
    dk = addrs(10)[9]
    assert call_backward(D(), dv=dk + 64) == lt2.LT2_ERR_INVALID_ARGUMENT    # two gradients overlap
    assert call_backward(D(T=0)) == lt2.LT2_OK
