"""fp64 CPU oracle for the KDA gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The CUDA library never imports,
links or calls anything here, and nothing here imports the CUDA library.

The C source (``kda_oracle.c``) runs the recurrence one token at a time in
fp64 (pages: "22580: from GPT-2 to Kimi K3, explained", sections "DeltaNet,
or Fast Weight Programmers" (cached forward), "Gated Delta Net" (the decay
alpha) and "KDA / Kimi Linear" (one decay per key channel)):

    S' = Diag(exp(log_alpha_t)) S;  r = S'^T k_t;  d = beta_t (v_t - r)
    S  = S' + k_t d^T;              o_t = S^T q_t

Inputs of any float dtype (bf16, fp32, fp64) are widened exactly to fp64
before the call, so the oracle sees precisely the values the GPU sees.

Pins (tests/test_oracle_pins.py) tie it to what the pages and mathematics
fix: the no-change, overwrite/retrieval, clear and no-update invariants, the
unrolled Householder product form, the ungated and gated chunk algebra, and
split/resume equivalence.

Two further forms of the same recurrence (``kda_forward_ex``):
  * the gate: per key channel (KDA, section "KDA / Kimi Linear"), one scalar
    per head and token (section "Gated Delta Net": a data-dependent scalar
    between 0 and 1 that multiplies the whole previous state) or none
    (alpha = 1, the plain delta rule of "DeltaNet, or Fast Weight
    Programmers");
  * the input prologue of the cached forward in "DeltaNet, or Fast Weight
    Programmers": q and k pass through SiLU and are L2-normalised over the
    head dimension (F.normalize, i.e. divided by max(norm, 1e-12)), beta is
    the sigmoid of its projection; the gate is read as alpha = sigmoid(x) of
    its projection x (a value between 0 and 1), so log_alpha = log sigmoid(x).
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_kda_forward.argtypes = [
            dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            dp, dp, ctypes.c_int]
        lib.oracle_kda_forward.restype = ctypes.c_int
        lib.oracle_kda_backward.argtypes = [
            dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_kda_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    """Exact widening to a contiguous fp64 numpy array (torch or numpy in)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def kda_forward(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None,
                n_threads=None):
    """Run the recurrence over packed sequences.

    q, k, log_alpha: [T_total, H, dk]; v: [T_total, H, dv]; beta: [T_total, H];
    init_state: [N, H, dk, dv] or None (zeros); cu_seqlens: [N+1] or None
    (one sequence of T_total tokens). Batched inputs [B, T, H, d] are accepted
    and treated as B sequences of T tokens. Returns (o, final_state) in fp64,
    o shaped like v.
    """
    q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
    s0 = _f64(init_state)
    out_shape = v.shape
    if q.ndim == 4:  # [B, T, H, d] -> packed
        B, T = q.shape[:2]
        if cu_seqlens is None:
            cu_seqlens = np.arange(B + 1, dtype=np.int64) * T
        q, k, v, la = (x.reshape(B * T, *x.shape[2:]) for x in (q, k, v, la))
        b = b.reshape(B * T, -1)
    T_total, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T_total], dtype=np.int64)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n_seq = cu.shape[0] - 1
    if cu[-1] != T_total:
        raise ValueError("cu_seqlens[-1] must equal the number of tokens")
    for x, shp in ((k, (T_total, H, dk)), (la, (T_total, H, dk)),
                   (v, (T_total, H, dv)), (b, (T_total, H))):
        if x.shape != shp:
            raise ValueError("shape mismatch: %s vs %s" % (x.shape, shp))
    if s0 is not None and s0.shape != (n_seq, H, dk, dv):
        raise ValueError("init_state must be [N, H, dk, dv]")
    o = np.zeros((T_total, H, dv), dtype=np.float64)
    fin = np.zeros((n_seq, H, dk, dv), dtype=np.float64)
    nt = default_threads() if n_threads is None else int(n_threads)
    rc = _load().oracle_kda_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        n_seq, H, dk, dv, _ptr(o), _ptr(fin), nt)
    if rc != 0:
        raise RuntimeError("oracle_kda_forward failed with code %d" % rc)
    return o.reshape(out_shape), fin


def kda_backward(q, k, v, log_alpha, beta, d_o, init_state=None, d_final=None,
                 cu_seqlens=None, n_threads=None):
    """Reverse mode of kda_forward (same layouts): given dL/do (shaped like o)
    and dL/dS_final ([N, H, dk, dv] or None = 0), returns a dict with dq, dk,
    dlog_alpha (shaped like q), dv (like v), dbeta (like beta) and d_init
    ([N, H, dk, dv]), all fp64."""
    q, k, v, la, b, g_o = map(_f64, (q, k, v, log_alpha, beta, d_o))
    s0, g_f = _f64(init_state), _f64(d_final)
    shapes = dict(q=q.shape, v=v.shape, b=b.shape)
    if q.ndim == 4:
        B, T = q.shape[:2]
        if cu_seqlens is None:
            cu_seqlens = np.arange(B + 1, dtype=np.int64) * T
        q, k, v, la, g_o = (x.reshape(B * T, *x.shape[2:]) for x in (q, k, v, la, g_o))
        b = b.reshape(B * T, -1)
    T_total, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T_total], dtype=np.int64)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n_seq = cu.shape[0] - 1
    if cu[-1] != T_total or g_o.shape != (T_total, H, dv):
        raise ValueError("shape mismatch")
    out = {n: np.zeros((T_total, H, dk)) for n in ("dq", "dk", "dlog_alpha")}
    out["dv"] = np.zeros((T_total, H, dv))
    out["dbeta"] = np.zeros((T_total, H))
    out["d_init"] = np.zeros((n_seq, H, dk, dv))
    nt = default_threads() if n_threads is None else int(n_threads)
    rc = _load().oracle_kda_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n_seq, H, dk, dv,
        _ptr(g_o), _ptr(g_f), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
        _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]), _ptr(out["d_init"]), nt)
    if rc != 0:
        raise RuntimeError("oracle_kda_backward failed with code %d" % rc)
    for n in ("dq", "dk", "dlog_alpha"):
        out[n] = out[n].reshape(shapes["q"])
    out["dv"] = out["dv"].reshape(shapes["v"])
    out["dbeta"] = out["dbeta"].reshape(shapes["b"])
    return out


# ---------------------------------------------------------------------------
# Gate forms and input prologue (plain fp64 numpy, elementwise definitions)
# ---------------------------------------------------------------------------

GATES = ("channel", "scalar", "none")


def expand_gate(log_alpha, gate, tok_head_shape, dk):
    """The per-key-channel log-decay a gate form stands for, [..., H, dk].

    channel: log_alpha is already [..., H, dk].
    scalar:  log_alpha is [..., H]; the one decay multiplies the whole state,
             i.e. the same value on every key channel.
    none:    alpha = 1 (log_alpha = 0); the argument is ignored.
    """
    if gate == "channel":
        la = _f64(log_alpha)
        if la.shape != tuple(tok_head_shape) + (dk,):
            raise ValueError("channel gate must be %s" % ((tuple(tok_head_shape) + (dk,)),))
        return la
    if gate == "scalar":
        la = _f64(log_alpha)
        if la.shape != tuple(tok_head_shape):
            raise ValueError("scalar gate must be %s" % (tuple(tok_head_shape),))
        return np.repeat(la[..., None], dk, axis=-1)
    if gate == "none":
        return np.zeros(tuple(tok_head_shape) + (dk,))
    raise ValueError("gate must be one of %s" % (GATES,))


def silu(x):
    """x * sigmoid(x)."""
    x = _f64(x)
    return x * sigmoid(x)


def sigmoid(x):
    """1 / (1 + exp(-x)), evaluated without overflow for either sign."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def log_sigmoid(x):
    """log(sigmoid(x)) = -log(1 + exp(-x)), evaluated without overflow."""
    x = _f64(x)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def l2_normalize(x, eps=1e-12):
    """x / max(||x||_2, eps) over the last axis."""
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def prologue_qk(x):
    """A query or key vector from its raw projection: L2-normalised SiLU."""
    return l2_normalize(silu(x))


def kda_forward_ex(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *,
                   gate="channel", raw_qk=False, raw_beta=False, raw_gate=False,
                   n_threads=None):
    """kda_forward with a gate form and an optional input prologue.

    gate: "channel" (log_alpha [..., H, dk]), "scalar" (log_alpha [..., H]) or
    "none" (log_alpha ignored). raw_qk: q and k are raw projections and go
    through prologue_qk; raw_beta: beta holds logits (sigmoid applied);
    raw_gate: log_alpha holds gate logits x and the decay is log sigmoid(x).
    The prologue is applied in fp64 before the token loop.
    """
    q, k = _f64(q), _f64(k)
    if raw_qk:
        q, k = prologue_qk(q), prologue_qk(k)
    b = _f64(beta)
    if raw_beta:
        b = sigmoid(b)
    la = None
    if gate != "none":
        la = _f64(log_alpha)
        if raw_gate:
            la = log_sigmoid(la)
    la = expand_gate(la, gate, q.shape[:-1], q.shape[-1])
    return kda_forward(q, k, v, la, b, init_state=init_state, cu_seqlens=cu_seqlens,
                       n_threads=n_threads)


def kda_decode_step(q, k, v, log_alpha, beta, state):
    """One decode step for B sequences: q, k, log_alpha [B, H, dk]; v [B, H, dv];
    beta [B, H]; state [B, H, dk, dv]. Returns (o [B, H, dv], new state)."""
    q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return kda_forward(q, k, v, la, b, init_state=state, cu_seqlens=cu)


def _prologue_qk_vjp(x, g, eps=1e-12):
    """Vector-Jacobian product of prologue_qk at the raw projection x with the
    cotangent g (both [..., d]): with s = sigmoid(x), u = x s (SiLU), r = ||u||
    and n = u / max(r, eps), the normalisation's Jacobian is (I - n n^T) / r
    when r > eps and I / eps otherwise, and SiLU's derivative is
    s (1 + x (1 - s))."""
    x, g = _f64(x), _f64(g)
    s = sigmoid(x)
    u = x * s
    r = np.sqrt(np.sum(u * u, axis=-1, keepdims=True))
    n = u / np.maximum(r, eps)
    du = np.where(r > eps, (g - n * np.sum(n * g, axis=-1, keepdims=True)) / np.maximum(r, eps),
                  g / eps)
    return du * s * (1.0 + x * (1.0 - s))


def kda_backward_ex(q, k, v, log_alpha, beta, d_o, init_state=None, d_final=None,
                    cu_seqlens=None, *, gate="channel", raw_qk=False, raw_beta=False,
                    raw_gate=False, n_threads=None):
    """Reverse mode of kda_forward_ex: the gradients with respect to the inputs
    as given (raw projections and logits when the prologue flags are set).

    The prologue is applied in fp64 as in kda_forward_ex, kda_backward gives
    the gradients with respect to the transformed inputs, and the chain rule
    takes them back through the prologue's elementwise definitions:
    dq, dk through _prologue_qk_vjp; dbeta times sigmoid'(x) = s (1 - s);
    dlog_alpha (summed over the key channels for the scalar gate) times
    d log sigmoid(x) / dx = sigmoid(-x). With gate "none", dlog_alpha is None.
    """
    q0, k0 = _f64(q), _f64(k)
    qn, kn = (prologue_qk(q0), prologue_qk(k0)) if raw_qk else (q0, k0)
    b0 = _f64(beta)
    b = sigmoid(b0) if raw_beta else b0
    la_in = None
    la = None
    if gate != "none":
        la_in = _f64(log_alpha)
        la = log_sigmoid(la_in) if raw_gate else la_in
    la = expand_gate(la, gate, qn.shape[:-1], qn.shape[-1])
    g = kda_backward(qn, kn, v, la, b, d_o, init_state=init_state, d_final=d_final,
                     cu_seqlens=cu_seqlens, n_threads=n_threads)
    if raw_qk:
        g["dq"] = _prologue_qk_vjp(q0, g["dq"])
        g["dk"] = _prologue_qk_vjp(k0, g["dk"])
    if raw_beta:
        s = sigmoid(b0)
        g["dbeta"] = g["dbeta"] * s * (1.0 - s)
    if gate == "none":
        g["dlog_alpha"] = None
    else:
        if gate == "scalar":
            g["dlog_alpha"] = g["dlog_alpha"].sum(-1)
        if raw_gate:
            g["dlog_alpha"] = g["dlog_alpha"] * sigmoid(-la_in)
    return g
