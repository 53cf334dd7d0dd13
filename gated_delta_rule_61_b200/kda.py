"""Python binding of libkda.so (ctypes). Argument marshalling only: every step
of the recurrence runs in the library's CUDA kernels; there is no fallback.

The C ABI (include/kda.h) takes device pointers; these wrappers take torch
CUDA tensors, check shapes and dtypes, pass ``data_ptr()`` values and the
current CUDA stream, and raise ``KdaError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

# Status codes and dtype codes of include/kda.h.
KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, \
    KDA_ERR_TIMEOUT = range(6)
KDA_F32, KDA_BF16 = 0, 1
KDA_GATE_CHANNEL, KDA_GATE_SCALAR, KDA_GATE_NONE = 0, 1, 2
KDA_RAW_QK, KDA_RAW_BETA, KDA_RAW_GATE = 1, 2, 4
GATES = {"channel": KDA_GATE_CHANNEL, "scalar": KDA_GATE_SCALAR, "none": KDA_GATE_NONE}
CHUNK_LOG_ALPHA_MIN = -10.0
DECODE_MAX_TOKENS = 16

EXPORTS = ("kda_status_string", "kda_version", "kda_prefill_workspace_bytes",
           "kda_prefill", "kda_prefill_ex", "kda_decode_step", "kda_decode_ex",
           "kda_backward_workspace_bytes", "kda_backward", "kda_backward_ex",
           "kda_prefill_noalloc",
           "kda_get_device_status", "kda_selftest_wait_timeout")
NOALLOC_MAX_SEQS = 65536


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


_lib = None


def lib():
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libkda.so is missing: build it with "
                           "`python -m gated_delta_rule_61_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, fp, ip, i32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    L.kda_status_string.argtypes = [ctypes.c_int]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    L.kda_version.restype = ctypes.c_int
    L.kda_prefill_workspace_bytes.argtypes = [ctypes.c_int] * 7
    L.kda_prefill_workspace_bytes.restype = ctypes.c_size_t
    L.kda_prefill.argtypes = [vp, vp, vp, fp, fp, fp, i32p, ip, ip, ip, ip, ip, ip,
                              ctypes.c_int, ctypes.c_int, vp, fp, vp, ctypes.c_size_t, vp]
    L.kda_prefill.restype = ctypes.c_int
    L.kda_prefill_ex.argtypes = [vp, vp, vp, fp, fp, fp, i32p, ip, ip, ip, ip, ip, ip,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_uint, ctypes.c_int, vp, fp,
                                 vp, ctypes.c_size_t, vp]
    L.kda_prefill_ex.restype = ctypes.c_int
    L.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, ip, ip, ip, ip, ctypes.c_int, vp, vp]
    L.kda_decode_step.restype = ctypes.c_int
    L.kda_decode_ex.argtypes = [vp, vp, vp, fp, fp, fp, ip, ip, ip, ip, ip, ctypes.c_int,
                                ctypes.c_int, ctypes.c_uint, vp, vp]
    L.kda_decode_ex.restype = ctypes.c_int
    L.kda_backward_workspace_bytes.argtypes = [ip, ctypes.c_int64, ip, ip, ip]
    L.kda_backward_workspace_bytes.restype = ctypes.c_size_t
    L.kda_backward.argtypes = [vp, vp, vp, fp, fp, fp, i32p, ip, ip, ip, ip, ip, ip,
                               ctypes.c_int, ctypes.c_int, vp, fp, fp, fp, fp, fp, fp, fp,
                               vp, ctypes.c_size_t, vp]
    L.kda_backward.restype = ctypes.c_int
    L.kda_backward_ex.argtypes = [vp, vp, vp, fp, fp, fp, i32p, ip, ip, ip, ip, ip, ip,
                                  ctypes.c_int, ctypes.c_int, ctypes.c_uint, vp, fp, fp, fp, fp,
                                  fp, fp, fp, vp, ctypes.c_size_t, vp]
    L.kda_backward_ex.restype = ctypes.c_int
    L.kda_prefill_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, i32p, ip, ip, ip, vp, fp, vp]
    L.kda_prefill_noalloc.restype = ctypes.c_int
    L.kda_get_device_status.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int), vp]
    L.kda_get_device_status.restype = ctypes.c_int
    L.kda_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    L.kda_selftest_wait_timeout.restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _check(t, name, shape, dtype, device):
    if t.device != device:
        raise ValueError("%s must be on %s" % (name, device))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def workspace_bytes(n_seq: int, H: int, dk: int, dv: int, dtype_code: int, chunk: int,
                    has_cu_seqlens: bool) -> int:
    """Bytes of workspace kda_prefill needs (see include/kda.h)."""
    return int(lib().kda_prefill_workspace_bytes(int(n_seq), int(H), int(dk), int(dv),
                                                 int(dtype_code), int(chunk),
                                                 1 if has_cu_seqlens else 0))


def _flags(raw_qk, raw_beta, raw_gate):
    return ((KDA_RAW_QK if raw_qk else 0) | (KDA_RAW_BETA if raw_beta else 0)
            | (KDA_RAW_GATE if raw_gate else 0))


def _gate_shape(gate, tok_head):
    if gate == "channel":
        return None
    return tuple(tok_head)


def prefill(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *, chunk=64,
            gate="channel", raw_qk=False, raw_beta=False, raw_gate=False,
            output_final_state=True, o=None, final_state=None, workspace=None, stream=None):
    """Chunked (chunk=64) or token-recurrent (chunk=0) KDA prefill.

    q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    log_alpha [B, T, H, dk] (gate "channel"), [B, T, H] ("scalar") or None
    ("none"); init_state [N, H, dk, dv] or None; cu_seqlens int32 [N+1]
    (then B = 1). raw_qk / raw_beta / raw_gate: the inputs are raw
    projections and the kernel applies the prologue (see kda_prefill_ex).
    Returns (o [B, T, H, dv] in q's dtype, final_state [N, H, dk, dv] fp32 or
    None).
    """
    if gate not in GATES:
        raise ValueError("gate must be one of %s" % list(GATES))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    dt = q.dtype
    code = _dtype_code(q)
    n_seq = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(k, "k", (B, T, H, dk), dt, dev)
    _check(v, "v", (B, T, H, dv), dt, dev)
    if gate == "channel":
        _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    elif gate == "scalar":
        _check(log_alpha, "log_alpha", (B, T, H), torch.float32, dev)
    else:
        log_alpha = None
    _check(beta, "beta", (B, T, H), torch.float32, dev)
    if init_state is not None:
        _check(init_state, "init_state", (n_seq, H, dk, dv), torch.float32, dev)
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("packed sequences (cu_seqlens) need B == 1")
        _check(cu_seqlens, "cu_seqlens", (n_seq + 1,), torch.int32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if output_final_state and final_state is None:
        final_state = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _check(final_state, "final_state", (n_seq, H, dk, dv), torch.float32, dev)
    need = workspace_bytes(n_seq, H, dk, dv, code, chunk, cu_seqlens is not None)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), int(n_seq), int(B), int(T), int(H), int(dk), int(dv), code,
        GATES[gate], _flags(raw_qk, raw_beta, raw_gate), int(chunk), _ptr(o),
        _ptr(final_state), _ptr(workspace), ws_bytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_ex")
    return o, final_state


def backward(q, k, v, log_alpha, beta, d_o, init_state=None, cu_seqlens=None, d_final=None,
             *, gate="channel", raw_qk=False, raw_beta=False, raw_gate=False, workspace=None,
             stream=None):
    """Gradients through the recurrence (kda_backward_ex): returns a dict of
    fp32 tensors dq, dk, dv, dlog_alpha (None for gate "none"), dbeta and
    d_init ([N, H, dk, dv]). Inputs as for prefill, including the prologue
    flags (the gradients are then with respect to the raw projections and
    logits); d_o shaped like v in v's dtype; d_final [N, H, dk, dv] fp32 or
    None."""
    if gate not in GATES:
        raise ValueError("gate must be one of %s" % list(GATES))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    n_seq = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    for t, name, shape, dtype in ((q, "q", (B, T, H, dk), dt), (k, "k", (B, T, H, dk), dt),
                                  (v, "v", (B, T, H, dv), dt), (d_o, "d_o", (B, T, H, dv), dt),
                                  (beta, "beta", (B, T, H), torch.float32)):
        _check(t, name, shape, dtype, dev)
    if gate == "channel":
        _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    elif gate == "scalar":
        _check(log_alpha, "log_alpha", (B, T, H), torch.float32, dev)
    else:
        log_alpha = None
    for t, name in ((init_state, "init_state"), (d_final, "d_final")):
        if t is not None:
            _check(t, name, (n_seq, H, dk, dv), torch.float32, dev)
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("packed sequences (cu_seqlens) need B == 1")
        _check(cu_seqlens, "cu_seqlens", (n_seq + 1,), torch.int32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty(B, T, H, dk, **f32), dk=torch.empty(B, T, H, dk, **f32),
               dv=torch.empty(B, T, H, dv, **f32), dbeta=torch.empty(B, T, H, **f32),
               d_init=torch.empty(n_seq, H, dk, dv, **f32))
    out["dlog_alpha"] = (None if gate == "none" else torch.empty(log_alpha.shape, **f32))
    need = int(lib().kda_backward_workspace_bytes(int(n_seq), int(B * T), int(H), int(dk),
                                                  int(dv)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().kda_backward_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), int(n_seq), int(B), int(T), int(H), int(dk), int(dv), code,
        GATES[gate], _flags(raw_qk, raw_beta, raw_gate), _ptr(d_o), _ptr(d_final),
        _ptr(out["dq"]), _ptr(out["dk"]),
        _ptr(out["dv"]), _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]), _ptr(out["d_init"]),
        _ptr(workspace), ws_bytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_backward_ex")
    return out


def prefill_noalloc(q, k, v, log_alpha, beta, cu_seqlens, init_state=None, *,
                    output_final_state=True, o=None, final_state=None, stream=None):
    """Packed variable-length chunked prefill that allocates no device memory
    inside the library (its scratch is a fixed array in libkda.so; see
    kda_prefill_noalloc in include/kda.h for the limits and the sharing rule).
    q, k, log_alpha [1, T, H, 128]; v [1, T, H, 128] (bf16); beta [1, T, H];
    cu_seqlens int32 [N+1]; init_state [N, H, 128, 128] fp32 or None.
    Returns (o, final_state). Output tensors are allocated here by torch
    unless passed in; pass o and final_state to keep the call allocation-free."""
    B, T, H, dk = q.shape
    dev = q.device
    n_seq = cu_seqlens.shape[0] - 1
    if B != 1 or dk != 128 or v.shape[-1] != 128 or q.dtype != torch.bfloat16:
        raise ValueError("prefill_noalloc takes packed bf16 inputs [1, T, H, 128]")
    for t, name, shape, dtype in ((q, "q", (1, T, H, 128), torch.bfloat16),
                                  (k, "k", (1, T, H, 128), torch.bfloat16),
                                  (v, "v", (1, T, H, 128), torch.bfloat16),
                                  (log_alpha, "log_alpha", (1, T, H, 128), torch.float32),
                                  (beta, "beta", (1, T, H), torch.float32),
                                  (cu_seqlens, "cu_seqlens", (n_seq + 1,), torch.int32)):
        _check(t, name, shape, dtype, dev)
    if init_state is not None:
        _check(init_state, "init_state", (n_seq, H, 128, 128), torch.float32, dev)
    if o is None:
        o = torch.empty((1, T, H, 128), dtype=torch.bfloat16, device=dev)
    else:
        _check(o, "o", (1, T, H, 128), torch.bfloat16, dev)
    if output_final_state and final_state is None:
        final_state = torch.empty((n_seq, H, 128, 128), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _check(final_state, "final_state", (n_seq, H, 128, 128), torch.float32, dev)
    st = lib().kda_prefill_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), int(n_seq), int(T), int(H), _ptr(o), _ptr(final_state),
        _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_noalloc")
    return o, final_state


def decode(q, k, v, log_alpha, beta, state, *, gate="channel", raw_qk=False, raw_beta=False,
           raw_gate=False, o=None, stream=None):
    """T tokens per sequence (1 <= T <= 16) against the cached ``state``
    [B, H, dk, dv] fp32, updated in place (one read and one write of it).
    q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H]; log_alpha
    [B, T, H, dk] / [B, T, H] / None per ``gate``. Returns o [B, T, H, dv]."""
    if gate not in GATES:
        raise ValueError("gate must be one of %s" % list(GATES))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(k, "k", (B, T, H, dk), dt, dev)
    _check(v, "v", (B, T, H, dv), dt, dev)
    if gate == "channel":
        _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    elif gate == "scalar":
        _check(log_alpha, "log_alpha", (B, T, H), torch.float32, dev)
    else:
        log_alpha = None
    _check(beta, "beta", (B, T, H), torch.float32, dev)
    _check(state, "state", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    st = lib().kda_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                             _ptr(state), int(B), int(T), int(H), int(dk), int(dv), code,
                             GATES[gate], _flags(raw_qk, raw_beta, raw_gate), _ptr(o),
                             _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_ex")
    return o


def decode_step(q, k, v, log_alpha, beta, state, *, o=None, stream=None):
    """One decode token per sequence; ``state`` [B, H, dk, dv] fp32 is
    updated in place. Returns o [B, H, dv] in q's dtype."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(q, "q", (B, H, dk), dt, dev)
    _check(k, "k", (B, H, dk), dt, dev)
    _check(v, "v", (B, H, dv), dt, dev)
    _check(log_alpha, "log_alpha", (B, H, dk), torch.float32, dev)
    _check(beta, "beta", (B, H), torch.float32, dev)
    _check(state, "state", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, H, dv), dt, dev)
    st = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                               _ptr(state), int(B), int(H), int(dk), int(dv), code, _ptr(o),
                               _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step")
    return o


def device_status(reset: bool = True, stream=None):
    """(status, detail) of the device status word; synchronises the stream."""
    detail = ctypes.c_int(0)
    st = lib().kda_get_device_status(1 if reset else 0, ctypes.byref(detail), _stream(stream))
    return int(st), int(detail.value)


def selftest_wait_timeout(max_ns: int = 2_000_000, stream=None):
    """Run the bounded-wait failure path on purpose (see
    kda_selftest_wait_timeout in include/kda.h); returns the launch status.
    Read the recorded timeout with device_status()."""
    return int(lib().kda_selftest_wait_timeout(int(max_ns), _stream(stream)))
