"""Python binding of liblt2gdr.so, the B200 looped gated-delta-rule mixer.

Thin ctypes layer over the C ABI of include/lt2_gdr.h with the same names
(lt2_gdr_prefill, lt2_gdr_decode, lt2_gdr_prefill_workspace_bytes, lt2_gdr_last_device_error,
lt2_status_string).  It only marshals arguments: torch tensors are passed as raw device
pointers together with the current CUDA stream, and every step of the computation runs in
the library's kernels.  ``prefill`` and ``decode`` are conveniences that allocate outputs
with torch and raise on a non-OK status.

The shared library is loaded on first use; if it is missing the call raises (there is no
fallback implementation).
"""
import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblt2gdr.so")

LT2_OK = 0
LT2_ERR_INVALID_ARGUMENT = 1
LT2_ERR_UNSUPPORTED = 2
LT2_ERR_WORKSPACE = 3
LT2_ERR_CUDA = 4
LT2_ERR_DEVICE_TIMEOUT = 5
LT2_ERR_RANGE = 6
LT2_ERR_DEVICE_CHECK = 7
LT2_ERR_SEQLENS = 8

LT2_DTYPE_F32 = 0
LT2_DTYPE_BF16 = 1
LT2_GATE_SCALAR = 0
LT2_GATE_PER_KEY = 1
LT2_GATE_PER_KEY_DECAY_FIRST = 2
LT2_ALGO_AUTO = 0
LT2_ALGO_TENSOR_CORE = 1
LT2_ALGO_CUDA_CORE = 2
LT2_OUT_SAME = 0
LT2_OUT_F32 = 1
LT2_OUT_BF16 = 2

# Every symbol include/lt2_gdr.h declares.
EXPORTS = (
    "lt2_gdr_prefill_workspace_bytes",
    "lt2_gdr_prefill",
    "lt2_gdr_prefill_fused",
    "lt2_gdr_decode",
    "lt2_gdr_decode_fused",
    "lt2_gdr_prefill_varlen",
    "lt2_gdr_backward_workspace_bytes",
    "lt2_gdr_backward",
    "lt2_gdr_backward_static",
    "lt2_swa_prefill",
    "lt2_gdr_last_device_error",
    "lt2_status_string",
    "lt2_last_cuda_error_string",
    "lt2_gdr_version",
)


class lt2_gdr_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("B", ctypes.c_int64), ("H", ctypes.c_int64),
                ("L", ctypes.c_int64), ("dk", ctypes.c_int64), ("dv", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("gate", ctypes.c_int32), ("algo", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32)]


class lt2_gdr_fused(ctypes.Structure):
    """The fused prologue and output gate (include/lt2_gdr.h); all zero selects none."""
    _fields_ = [("qk_l2norm", ctypes.c_int32), ("gate_logits", ctypes.c_int32),
                ("alpha_scale", ctypes.c_float), ("reserved", ctypes.c_int32),
                ("z", ctypes.c_void_p)]


class lt2_swa_dims(ctypes.Structure):
    """Sizes of a sliding-window attention prefill (include/lt2_gdr.h)."""
    _fields_ = [("T", ctypes.c_int64), ("B", ctypes.c_int64), ("H", ctypes.c_int64),
                ("L", ctypes.c_int64), ("d", ctypes.c_int64), ("window", ctypes.c_int64),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int32), ("algo", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32)]


def make_fused(qk_l2norm=False, gate_logits=False, alpha_scale=1.0, z=None):
    """An lt2_gdr_fused; ``z`` is a tensor (its data pointer is taken), an address or None."""
    return lt2_gdr_fused(int(bool(qk_l2norm)), int(bool(gate_logits)), float(alpha_scale), 0, _p(z))


class Lt2Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        extra = ""
        if status == LT2_ERR_CUDA:
            extra = ": " + lib().lt2_last_cuda_error_string().decode()
        super().__init__(f"{where} returned {lt2_status_string(status)}{extra}")


_LIB = None


def lib():
    """The loaded liblt2gdr.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m gated_delta_rule_looped_b200.build` (no fallback exists)")
        _LIB = load_library(LIB_PATH)
    return _LIB


def load_library(path):
    """A build of the library at ``path`` with the argument types of include/lt2_gdr.h declared
    (the tests load the debug build, liblt2gdr_debug.so, this way; it also declares the hooks of
    include/lt2_gdr_debug.h when the build exports them, and loads builds that predate the fused
    entry points)."""
    L = ctypes.CDLL(path)
    vp, fp = ctypes.c_void_p, ctypes.c_void_p
    dims_p = ctypes.POINTER(lt2_gdr_dims)
    L.lt2_gdr_prefill_workspace_bytes.argtypes = [dims_p]
    L.lt2_gdr_prefill_workspace_bytes.restype = ctypes.c_size_t
    L.lt2_gdr_prefill.argtypes = [dims_p, vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                  ctypes.c_size_t, vp]
    L.lt2_gdr_prefill.restype = ctypes.c_int
    L.lt2_gdr_decode.argtypes = [dims_p, vp, vp, vp, fp, fp, fp, vp, vp]
    L.lt2_gdr_decode.restype = ctypes.c_int
    if hasattr(L, "lt2_gdr_prefill_fused"):
        fused_p = ctypes.POINTER(lt2_gdr_fused)
        L.lt2_gdr_prefill_fused.argtypes = [dims_p, fused_p, vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                            ctypes.c_size_t, vp]
        L.lt2_gdr_prefill_fused.restype = ctypes.c_int
        L.lt2_gdr_decode_fused.argtypes = [dims_p, fused_p, vp, vp, vp, fp, fp, fp, vp, vp]
        L.lt2_gdr_decode_fused.restype = ctypes.c_int
    if hasattr(L, "lt2_gdr_prefill_varlen"):
        L.lt2_gdr_prefill_varlen.argtypes = [dims_p, ctypes.POINTER(lt2_gdr_fused), vp, vp, vp, vp, fp, fp, fp, vp,
                                             fp, vp, ctypes.c_size_t, vp]
        L.lt2_gdr_prefill_varlen.restype = ctypes.c_int
    if hasattr(L, "lt2_gdr_backward"):
        L.lt2_gdr_backward_workspace_bytes.argtypes = [dims_p]
        L.lt2_gdr_backward_workspace_bytes.restype = ctypes.c_size_t
        L.lt2_gdr_backward.argtypes = [dims_p, vp, vp, vp, fp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp, vp,
                                       ctypes.c_size_t, vp]
        L.lt2_gdr_backward.restype = ctypes.c_int
    if hasattr(L, "lt2_gdr_backward_static"):
        L.lt2_gdr_backward_static.argtypes = [dims_p, vp, vp, vp, fp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp, vp]
        L.lt2_gdr_backward_static.restype = ctypes.c_int
    if hasattr(L, "lt2_swa_prefill"):
        L.lt2_swa_prefill.argtypes = [ctypes.POINTER(lt2_swa_dims), vp, vp, vp, vp, vp]
        L.lt2_swa_prefill.restype = ctypes.c_int
    L.lt2_gdr_last_device_error.argtypes = []
    L.lt2_gdr_last_device_error.restype = ctypes.c_int
    L.lt2_status_string.argtypes = [ctypes.c_int]
    L.lt2_status_string.restype = ctypes.c_char_p
    L.lt2_last_cuda_error_string.argtypes = []
    L.lt2_last_cuda_error_string.restype = ctypes.c_char_p
    L.lt2_gdr_version.argtypes = []
    L.lt2_gdr_version.restype = ctypes.c_int
    if hasattr(L, "lt2_debug_set_skip_chunk"):
        L.lt2_debug_set_skip_chunk.argtypes = [ctypes.c_int, ctypes.c_int]
        L.lt2_debug_set_skip_chunk.restype = ctypes.c_int
        L.lt2_debug_wait_timeout_ns.argtypes = []
        L.lt2_debug_wait_timeout_ns.restype = ctypes.c_uint64
    return L


def make_dims(T, B, H, L, dk, dv, dtype=LT2_DTYPE_BF16, gate=LT2_GATE_SCALAR,
              algo=LT2_ALGO_AUTO, out_dtype=LT2_OUT_SAME):
    return lt2_gdr_dims(T, B, H, L, dk, dv, dtype, gate, algo, out_dtype)


def _p(x):
    """Raw pointer of a tensor (or None / an int address passed through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --- the C ABI, same names ---------------------------------------------------------------

def lt2_gdr_prefill_workspace_bytes(dims):
    return lib().lt2_gdr_prefill_workspace_bytes(ctypes.byref(dims))


def lt2_gdr_prefill(dims, q, k, v, alpha, beta, S0, o, S_out, workspace=None,
                    workspace_bytes=0, stream=None):
    return lib().lt2_gdr_prefill(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(alpha), _p(beta),
                                 _p(S0), _p(o), _p(S_out), _p(workspace), int(workspace_bytes),
                                 _stream(stream))


def lt2_gdr_decode(dims, q, k, v, alpha, beta, S, o, stream=None):
    return lib().lt2_gdr_decode(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(alpha), _p(beta),
                                _p(S), _p(o), _stream(stream))


def lt2_gdr_prefill_fused(dims, fused, q, k, v, alpha, beta, S0, o, S_out, workspace=None,
                          workspace_bytes=0, stream=None):
    return lib().lt2_gdr_prefill_fused(ctypes.byref(dims), None if fused is None else ctypes.byref(fused),
                                       _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(o),
                                       _p(S_out), _p(workspace), int(workspace_bytes), _stream(stream))


def lt2_gdr_decode_fused(dims, fused, q, k, v, alpha, beta, S, o, stream=None):
    return lib().lt2_gdr_decode_fused(ctypes.byref(dims), None if fused is None else ctypes.byref(fused),
                                      _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S), _p(o),
                                      _stream(stream))


def lt2_gdr_prefill_varlen(dims, fused, cu_seqlens, q, k, v, alpha, beta, S0, o, S_out, workspace=None,
                           workspace_bytes=0, stream=None):
    return lib().lt2_gdr_prefill_varlen(ctypes.byref(dims), None if fused is None else ctypes.byref(fused),
                                        _p(cu_seqlens), _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(o),
                                        _p(S_out), _p(workspace), int(workspace_bytes), _stream(stream))


def lt2_gdr_backward_workspace_bytes(dims):
    return lib().lt2_gdr_backward_workspace_bytes(ctypes.byref(dims))


def lt2_gdr_backward(dims, q, k, v, alpha, beta, S0, dO, dS_L, dq, dk, dv, dalpha, dbeta, dS0, workspace=None,
                     workspace_bytes=0, stream=None):
    return lib().lt2_gdr_backward(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(dO),
                                  _p(dS_L), _p(dq), _p(dk), _p(dv), _p(dalpha), _p(dbeta), _p(dS0), _p(workspace),
                                  int(workspace_bytes), _stream(stream))


def lt2_gdr_backward_static(dims, q, k, v, alpha, beta, S0, dO, dS_L, dq, dk, dv, dalpha, dbeta, dS0,
                            stream=None):
    return lib().lt2_gdr_backward_static(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0),
                                         _p(dO), _p(dS_L), _p(dq), _p(dk), _p(dv), _p(dalpha), _p(dbeta),
                                         _p(dS0), _stream(stream))


def lt2_swa_prefill(dims, q, k, v, o, stream=None):
    return lib().lt2_swa_prefill(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(o), _stream(stream))


def lt2_gdr_last_device_error():
    return lib().lt2_gdr_last_device_error()


def lt2_status_string(status):
    return lib().lt2_status_string(int(status)).decode()


# --- conveniences on torch tensors ---------------------------------------------------------

_OUT = {None: LT2_OUT_SAME, "same": LT2_OUT_SAME, "f32": LT2_OUT_F32, "bf16": LT2_OUT_BF16}


def _out_torch_dtype(in_dtype, out):
    import torch
    if out in (None, "same"):
        return in_dtype
    return torch.float32 if out == "f32" else torch.bfloat16


def _gate(per_key, order):
    """lt2_gate for a gating and an order of the per-key factors ("delta_first", the equation
    as printed, or "decay_first"); the order does not matter for scalar gating."""
    if order not in ("delta_first", "decay_first"):
        raise ValueError(f"order must be 'delta_first' or 'decay_first', got {order!r}")
    if not per_key:
        return LT2_GATE_SCALAR
    return LT2_GATE_PER_KEY_DECAY_FIRST if order == "decay_first" else LT2_GATE_PER_KEY


def _dims_from(q, v, alpha, per_key, algo, out=None, order="delta_first"):
    import torch
    if q.dim() != 5 or v.dim() != 5:
        raise ValueError("q, k, v must be [T, B, H, L, d]")
    T, B, H, L, dk = q.shape
    dv = v.shape[-1]
    dt = {torch.float32: LT2_DTYPE_F32, torch.bfloat16: LT2_DTYPE_BF16}.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if per_key is None:
        per_key = alpha.dim() == 5
    return make_dims(T, B, H, L, dk, dv, dt, _gate(per_key, order), algo, _OUT[out])


def _check(name, t, shape, dtype, device):
    """A tensor handed to the library by pointer: on ``device``, contiguous, of the given shape
    and dtype (the C ABI reads raw row-major memory and cannot tell)."""
    if t is None:
        return
    if not hasattr(t, "is_cuda"):
        raise TypeError(f"{name} must be a torch tensor, got {type(t).__name__}")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _require_cuda(q):
    if not getattr(q, "is_cuda", False):
        raise ValueError(f"q must be a CUDA tensor, got {getattr(q, 'device', type(q).__name__)}")


def _check_call(q, k, v, alpha, beta, states, o, per_key, out):
    """Validate the tensors of a prefill ([T,B,H,L,d]) or decode ([T,B,H,d]) call: all on q's
    device, which must also be the current device (the library launches on the current one)."""
    import torch
    lead, dk, dv = tuple(q.shape[:-1]), q.shape[-1], v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError(f"q must be a CUDA tensor, got {dev}")
    if dev.index != torch.cuda.current_device():
        raise ValueError(f"q is on {dev} but the current device is cuda:{torch.cuda.current_device()}")
    _check("q", q, q.shape, q.dtype, dev)
    _check("k", k, q.shape, q.dtype, dev)
    _check("v", v, lead + (dv,), q.dtype, dev)
    _check("alpha", alpha, lead + ((dk,) if per_key else ()), torch.float32, dev)
    _check("beta", beta, lead, torch.float32, dev)
    for name, S in states:
        _check(name, S, tuple(q.shape[:3]) + (dk, dv), torch.float32, dev)
    _check("o", o, lead + (dv,), _out_torch_dtype(q.dtype, out), dev)


def prefill(q, k, v, alpha, beta, S0=None, per_key=None, algo=LT2_ALGO_AUTO, o=None,
            S_out=None, out=None, stream=None, order="delta_first", qk_l2norm=False,
            gate_logits=False, alpha_scale=1.0, z=None):
    """Run the looped prefill on CUDA tensors; returns (o, S_out).  ``out`` selects the
    storage type of o: None/"same" (as the inputs), "f32" or "bf16"; ``order`` the order of
    the per-key factors ("delta_first" as printed, or "decay_first").  ``qk_l2norm``,
    ``gate_logits``/``alpha_scale`` and ``z`` select the fused prologue and output gate
    (lt2_gdr_prefill_fused).  The call runs on the tensors' device (made current for its
    duration), on ``stream`` or that device's current stream."""
    import torch
    _require_cuda(q)
    fused = None
    if qk_l2norm or gate_logits or z is not None:
        fused = make_fused(qk_l2norm, gate_logits, alpha_scale, z)
    with torch.cuda.device(q.device):
        return _prefill(q, k, v, alpha, beta, S0, per_key, algo, o, S_out, out, stream, order, fused, z)


def _prefill(q, k, v, alpha, beta, S0, per_key, algo, o, S_out, out, stream, order, fused=None, z=None):
    import torch
    dims = _dims_from(q, v, alpha, per_key, algo, out, order)
    _check_call(q, k, v, alpha, beta, [("S0", S0), ("S_out", S_out)], o, dims.gate != LT2_GATE_SCALAR, out)
    _check("z", z, v.shape, q.dtype, q.device)
    if o is None:
        o = torch.empty(v.shape, dtype=_out_torch_dtype(q.dtype, out), device=v.device)
    if S_out is None:
        S_out = torch.empty(tuple(q.shape[:3]) + (q.shape[-1], v.shape[-1]),
                            dtype=torch.float32, device=q.device)
    ws_bytes = lt2_gdr_prefill_workspace_bytes(dims)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device) if ws_bytes else None
    if fused is None:
        st = lt2_gdr_prefill(dims, q, k, v, alpha, beta, S0, o, S_out, ws, ws_bytes, stream)
    else:
        st = lt2_gdr_prefill_fused(dims, fused, q, k, v, alpha, beta, S0, o, S_out, ws, ws_bytes, stream)
    if st != LT2_OK:
        raise Lt2Error(st, "lt2_gdr_prefill")
    return o, S_out


def decode(q, k, v, alpha, beta, S, per_key=None, o=None, out=None, stream=None, order="delta_first",
           qk_l2norm=False, gate_logits=False, alpha_scale=1.0, z=None):
    """One decode token per (loop, batch, head); q/k/v [T,B,H,d]; S updated in place.  The
    fused prologue and output gate as in ``prefill``.  Runs on the tensors' device (made
    current for the call)."""
    import torch
    _require_cuda(q)
    fused = None
    if qk_l2norm or gate_logits or z is not None:
        fused = make_fused(qk_l2norm, gate_logits, alpha_scale, z)
    with torch.cuda.device(q.device):
        return _decode(q, k, v, alpha, beta, S, per_key, o, out, stream, order, fused, z)


def _decode(q, k, v, alpha, beta, S, per_key, o, out, stream, order, fused=None, z=None):
    import torch
    per_key = (alpha.dim() == 4) if per_key is None else per_key
    T, B, H, dk = q.shape
    dv = v.shape[-1]
    dt = {torch.float32: LT2_DTYPE_F32, torch.bfloat16: LT2_DTYPE_BF16}[q.dtype]
    dims = make_dims(T, B, H, 1, dk, dv, dt, _gate(per_key, order), out_dtype=_OUT[out])
    _check_call(q, k, v, alpha, beta, [("S", S)], o, per_key, out)
    _check("z", z, v.shape, q.dtype, q.device)
    if o is None:
        o = torch.empty(v.shape, dtype=_out_torch_dtype(q.dtype, out), device=v.device)
    if fused is None:
        st = lt2_gdr_decode(dims, q, k, v, alpha, beta, S, o, stream)
    else:
        st = lt2_gdr_decode_fused(dims, fused, q, k, v, alpha, beta, S, o, stream)
    if st != LT2_OK:
        raise Lt2Error(st, "lt2_gdr_decode")
    return o


def swa_prefill(q, k, v, window, scale=None, algo=LT2_ALGO_AUTO, o=None, out=None, stream=None):
    """Sliding-window attention over [T, B, H, L, d] CUDA tensors (lt2_swa_prefill): every token
    attends to itself and the window - 1 tokens before it; ``scale`` multiplies q.k (None:
    1/sqrt(d)).  Returns o, of the inputs' dtype or ``out`` ("f32" / "bf16")."""
    import torch
    _require_cuda(q)
    if q.dim() != 5:
        raise ValueError("q, k, v must be [T, B, H, L, d]")
    dt = {torch.float32: LT2_DTYPE_F32, torch.bfloat16: LT2_DTYPE_BF16}.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if scale is not None and not scale > 0:
        raise ValueError("scale must be positive (None selects 1/sqrt(d))")
    with torch.cuda.device(q.device):
        dev = q.device
        for name, t in (("q", q), ("k", k), ("v", v)):
            _check(name, t, q.shape, q.dtype, dev)
        odt = _out_torch_dtype(q.dtype, out)
        _check("o", o, q.shape, odt, dev)
        if o is None:
            o = torch.empty(q.shape, dtype=odt, device=dev)
        T, B, H, L, d = q.shape
        dims = lt2_swa_dims(T, B, H, L, d, int(window), 0.0 if scale is None else float(scale), dt, algo, _OUT[out])
        st = lt2_swa_prefill(dims, q, k, v, o, stream)
        if st != LT2_OK:
            raise Lt2Error(st, "lt2_swa_prefill")
        return o


def prefill_varlen(q, k, v, alpha, beta, cu_seqlens, S0=None, per_key=None, algo=LT2_ALGO_AUTO, o=None,
                   S_out=None, out=None, stream=None, order="delta_first", qk_l2norm=False, gate_logits=False,
                   alpha_scale=1.0, z=None):
    """The looped prefill over packed sequences (lt2_gdr_prefill_varlen): q, k, v [T, H, Ntot, d],
    alpha [T, H, Ntot] (or [..., d] per key), beta [T, H, Ntot], cu_seqlens an int64 CUDA tensor of
    B + 1 offsets.  Returns (o [T, H, Ntot, d], S_out [T, B, H, d, d]); the other arguments as in
    ``prefill``."""
    import torch
    _require_cuda(q)
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [T, H, Ntot, d]")
    if cu_seqlens.dtype != torch.int64 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D int64 tensor of B + 1 offsets")
    fused = None
    if qk_l2norm or gate_logits or z is not None:
        fused = make_fused(qk_l2norm, gate_logits, alpha_scale, z)
    with torch.cuda.device(q.device):
        T, H, N, dk = q.shape
        dv = v.shape[-1]
        B = cu_seqlens.numel() - 1
        dt = {torch.float32: LT2_DTYPE_F32, torch.bfloat16: LT2_DTYPE_BF16}.get(q.dtype)
        if dt is None:
            raise ValueError(f"unsupported dtype {q.dtype}")
        if per_key is None:
            per_key = alpha.dim() == 4
        dims = make_dims(T, B, H, N, dk, dv, dt, _gate(per_key, order), algo, _OUT[out])
        dev = q.device
        _check("cu_seqlens", cu_seqlens, (B + 1,), torch.int64, dev)
        _check("k", k, q.shape, q.dtype, dev)
        _check("v", v, (T, H, N, dv), q.dtype, dev)
        _check("alpha", alpha, (T, H, N) + ((dk,) if per_key else ()), torch.float32, dev)
        _check("beta", beta, (T, H, N), torch.float32, dev)
        _check("z", z, (T, H, N, dv), q.dtype, dev)
        for name, S in (("S0", S0), ("S_out", S_out)):
            _check(name, S, (T, B, H, dk, dv), torch.float32, dev)
        odt = _out_torch_dtype(q.dtype, out)
        _check("o", o, (T, H, N, dv), odt, dev)
        if o is None:
            o = torch.empty((T, H, N, dv), dtype=odt, device=dev)
        if S_out is None:
            S_out = torch.empty((T, B, H, dk, dv), dtype=torch.float32, device=dev)
        st = lt2_gdr_prefill_varlen(dims, fused, cu_seqlens, q, k, v, alpha, beta, S0, o, S_out, None, 0, stream)
        if st != LT2_OK:
            raise Lt2Error(st, "lt2_gdr_prefill_varlen")
        return o, S_out


def backward(q, k, v, alpha, beta, dO, S0=None, dS_L=None, per_key=None, order="delta_first", stream=None):
    """Gradients of sum(dO * o) + sum(dS_L * S_out) of ``prefill`` (lt2_gdr_backward), fp32:
    returns a dict dq, dk, dv, dalpha, dbeta, dS0.  The workspace is allocated with torch."""
    import torch
    _require_cuda(q)
    with torch.cuda.device(q.device):
        dims = _dims_from(q, v, alpha, per_key, LT2_ALGO_AUTO, None, order)
        pk = dims.gate != LT2_GATE_SCALAR
        _check_call(q, k, v, alpha, beta, [("S0", S0), ("dS_L", dS_L)], None, pk, None)
        _check("dO", dO, v.shape, q.dtype, q.device)
        dev = q.device
        f32 = dict(dtype=torch.float32, device=dev)
        g = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(q.shape, **f32), "dv": torch.empty(v.shape, **f32),
             "dalpha": torch.empty(alpha.shape, **f32), "dbeta": torch.empty(beta.shape, **f32),
             "dS0": torch.empty(tuple(q.shape[:3]) + (q.shape[-1], v.shape[-1]), **f32)}
        ws_bytes = lt2_gdr_backward_workspace_bytes(dims)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
        st = lt2_gdr_backward(dims, q, k, v, alpha, beta, S0, dO, dS_L, g["dq"], g["dk"], g["dv"], g["dalpha"],
                              g["dbeta"], g["dS0"], ws, ws_bytes, stream)
        if st != LT2_OK:
            raise Lt2Error(st, "lt2_gdr_backward")
        return g


def prefill_host(q, k, v, alpha, beta, o, S_out, S0=None, per_key=None, order="delta_first", device=None,
                 slots=2):
    """The looped prefill on inputs that live in pinned host memory, with o and S_out written back
    to pinned host tensors: the loops run one at a time through ``slots`` device buffers on three
    streams, so that the host-to-device copy of loop tau + 1, the call on loop tau (lt2_gdr_prefill
    with T = 1) and the device-to-host copy of loop tau - 1 overlap (PCIe moves data both ways at
    once).  Device memory: ``slots`` loops' inputs and outputs.  The work is enqueued behind the
    current stream of ``device`` and that stream waits for all of it, so the caller synchronises as
    usual.  Shapes as in ``prefill``; q ... S_out are host tensors (pinned for the copies to
    overlap)."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    if q.is_cuda:
        raise ValueError("prefill_host takes host tensors; use prefill for device tensors")
    T = q.shape[0]
    with torch.cuda.device(dev):
        cur = torch.cuda.current_stream()
        s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        for st in (s_in, s_run, s_out):
            st.wait_stream(cur)
        ins = ("q", "k", "v", "alpha", "beta") + (("S0",) if S0 is not None else ())
        host = dict(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0)
        buf = [{n: torch.empty(host[n].shape[1:], dtype=host[n].dtype, device=dev) for n in ins} for _ in range(slots)]
        obuf = [(torch.empty(o.shape[1:], dtype=o.dtype, device=dev),
                 torch.empty(S_out.shape[1:], dtype=S_out.dtype, device=dev)) for _ in range(slots)]
        in_free = [None] * slots      # the call on the slot's previous loop is done with its inputs
        out_free = [None] * slots     # the slot's previous outputs have reached the host
        out_kind = "same" if o.dtype == q.dtype else ("f32" if o.dtype == torch.float32 else "bf16")
        for tau in range(T):
            sl = tau % slots
            with torch.cuda.stream(s_in):
                if in_free[sl] is not None:
                    s_in.wait_event(in_free[sl])
                for n in ins:
                    buf[sl][n].copy_(host[n][tau], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ready)
                if out_free[sl] is not None:
                    s_run.wait_event(out_free[sl])
                b = buf[sl]
                prefill(b["q"][None], b["k"][None], b["v"][None], b["alpha"][None], b["beta"][None],
                        S0=b["S0"][None] if S0 is not None else None, per_key=per_key, o=obuf[sl][0][None],
                        S_out=obuf[sl][1][None], out=out_kind, stream=s_run, order=order)
                done = torch.cuda.Event()
                done.record(s_run)
                in_free[sl] = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                o[tau].copy_(obuf[sl][0], non_blocking=True)
                S_out[tau].copy_(obuf[sl][1], non_blocking=True)
                back = torch.cuda.Event()
                back.record(s_out)
                out_free[sl] = back
        cur.wait_stream(s_out)
        cur.wait_stream(s_run)
        # the slot buffers stay alive until the streams are done with them
        for t in [x for b in buf for x in b.values()] + [x for pair in obuf for x in pair]:
            t.record_stream(s_in)
            t.record_stream(s_run)
            t.record_stream(s_out)
    return o, S_out
