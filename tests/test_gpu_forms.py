"""GPU parity of the gate forms, the fused input prologue and multi-token
decode, through the C ABI, against the fp64 oracle's kda_forward_ex.

Gate forms: per key channel (KDA), one scalar per token (Gated DeltaNet),
none (DeltaNet). Prologue: raw q/k projections (SiLU then L2 normalisation
in the kernel), beta logits (sigmoid), gate logits (log sigmoid). Each is run
on the chunked tensor-core kernel (in its one-CTA and ring launch shapes),
on the token-recurrent kernel and on the decode kernel. Tolerances as in
test_gpu_parity: bf16 path 1e-2 (o) and 5e-3 (state), fp32 path 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import decode_state
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, TOL_F32, assert_close

pytestmark = pytest.mark.gpu
CLAMP = kda.CHUNK_LOG_ALPHA_MIN


def _inputs(B, T, H, dk, dv, dtype, gate, raw, seed, init_std=0.1, lengths=None):
    """Seeded inputs of a prefill call. With raw=True, q/k are unnormalised
    N(0,1) projections, beta and the gate are logits (N(0,1) and N(3,1));
    otherwise q/k are unit vectors, beta = sigmoid, log_alpha = log sigmoid."""
    g = torch.Generator().manual_seed(seed)
    rn = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    n_seq = B if lengths is None else len(lengths)
    if lengths is not None:
        T = int(sum(lengths))
    q, k, v = rn(B, T, H, dk), rn(B, T, H, dk), rn(B, T, H, dv)
    if not raw:
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
    gshape = {"channel": (B, T, H, dk), "scalar": (B, T, H), "none": None}[gate]
    la = None
    if gshape is not None:
        x = rn(*gshape) + 3.0
        la = (x if raw else torch.nn.functional.logsigmoid(x)).float()
    b = rn(B, T, H)
    beta = (b if raw else torch.sigmoid(b)).float()
    s0 = None if init_std is None else (rn(n_seq, H, dk, dv) * init_std).float()
    cu = None
    if lengths is not None:
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), log_alpha=la, beta=beta,
                init_state=s0, cu_seqlens=cu)


def _oracle(inp, gate, raw, clamp):
    la = inp["log_alpha"]
    cu = inp["cu_seqlens"]
    names = ("q", "k", "v", "beta")
    if cu is not None:
        q, k, v, b = (inp[n][0] for n in names)
        la = None if la is None else la[0]
        cu = cu.numpy().astype(np.int64)
    else:
        q, k, v, b = (inp[n] for n in names)
    if la is not None:
        la = la.double()
        if raw:
            la = torch.from_numpy(oracle.log_sigmoid(la))
        if clamp:
            la = la.clamp(min=CLAMP)
    return oracle.kda_forward_ex(q, k, v, la, b, init_state=inp["init_state"], cu_seqlens=cu,
                                 gate=gate, raw_qk=raw, raw_beta=raw, raw_gate=False)


def _gpu(inp, gate, raw, chunk):
    g = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                       init_state=g["init_state"], cu_seqlens=g["cu_seqlens"], chunk=chunk,
                       gate=gate, raw_qk=raw, raw_beta=raw, raw_gate=raw)
    torch.cuda.synchronize()
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)
    return (o[0] if inp["cu_seqlens"] is not None else o), s


# B, T, H chosen for each launch shape of the chunked kernel on 148 SMs:
# 6 chains (ring of 4), 40 chains (ring of 2), 80 chains (one CTA per chain).
CHUNK_SHAPES = [(2, 200, 3), (1, 130, 40), (2, 97, 40)]


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("raw", [False, True])
@pytest.mark.parametrize("B,T,H", CHUNK_SHAPES)
def test_chunk_gate_forms_and_prologue(gate, raw, B, T, H):
    inp = _inputs(B, T, H, 128, 128, torch.bfloat16, gate, raw, seed=B * 100 + H + T)
    o_ref, s_ref = _oracle(inp, gate, raw, clamp=True)
    o, s = _gpu(inp, gate, raw, 64)
    what = "chunk gate=%s raw=%s" % (gate, raw)
    assert_close(o, o_ref, TOL_BF16_O, what + " o")
    assert_close(s, s_ref, TOL_BF16_STATE, what + " state")


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("raw", [False, True])
def test_chunk_forms_packed_sequences(gate, raw):
    inp = _inputs(1, 0, 4, 128, 128, torch.bfloat16, gate, raw, seed=7,
                  lengths=[0, 1, 63, 64, 65, 200, 17])
    o_ref, s_ref = _oracle(inp, gate, raw, clamp=True)
    o, s = _gpu(inp, gate, raw, 64)
    assert_close(o, o_ref, TOL_BF16_O, "packed o")
    assert_close(s, s_ref, TOL_BF16_STATE, "packed state")


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("raw", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_recurrent_gate_forms_and_prologue(gate, raw, dtype, dk, dv):
    inp = _inputs(2, 75, 3, dk, dv, dtype, gate, raw, seed=dk + dv + (7 if raw else 0))
    o_ref, s_ref = _oracle(inp, gate, raw, clamp=False)
    o, s = _gpu(inp, gate, raw, 0)
    tol_o = TOL_F32 if dtype == torch.float32 else TOL_BF16_O
    tol_s = TOL_F32 if dtype == torch.float32 else TOL_BF16_STATE
    assert_close(o, o_ref, tol_o, "recurrent o")
    assert_close(s, s_ref, tol_s, "recurrent state")


@pytest.mark.parametrize("strong", [False, True])
def test_scalar_gate_equals_broadcast_channel_gate_on_the_gpu(strong):
    """The same decay on every channel through the channel form gives the
    scalar form's result (same kernel arithmetic, bit for bit), also with
    strong decays (uniform in [-30, 0], some -inf) that the clamp reaches."""
    inp = _inputs(2, 150, 3, 128, 128, torch.bfloat16, "scalar", False, seed=5)
    if strong:
        g = torch.Generator().manual_seed(55)
        la = -30.0 * torch.rand(2, 150, 3, generator=g)
        la[torch.rand(2, 150, 3, generator=g) < 0.05] = -float("inf")
        inp["log_alpha"] = la.float()
    o1, s1 = _gpu(inp, "scalar", False, 64)
    inp2 = dict(inp)
    inp2["log_alpha"] = inp["log_alpha"][..., None].expand(2, 150, 3, 128).contiguous()
    o2, s2 = _gpu(inp2, "channel", False, 64)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_no_gate_equals_zero_channel_gate_on_the_gpu():
    """No decay through the specialised form equals log_alpha = 0 on every
    channel through the per-channel form, bit for bit (every factor is
    exactly 1 there)."""
    inp = _inputs(2, 150, 3, 128, 128, torch.bfloat16, "none", False, seed=6)
    o1, s1 = _gpu(inp, "none", False, 64)
    inp2 = dict(inp)
    inp2["log_alpha"] = torch.zeros(2, 150, 3, 128)
    o2, s2 = _gpu(inp2, "channel", False, 64)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


# ---------------------------------------------------------------------------
# Decode: T tokens per call against the cached state
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 2, 4, 7, 16])
@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("raw", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_multi_token_decode_against_oracle(T, gate, raw, dtype):
    B, H, d = 5, 3, 128
    inp = _inputs(B, T, H, d, d, dtype, gate, raw, seed=31 + T, init_std=None)
    S0 = decode_state(B, H, d, d, std=0.05, seed=T)
    inp["init_state"] = S0
    o_ref, s_ref = _oracle(inp, gate, raw, clamp=False)
    g = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    S = S0.cuda()
    o = kda.decode(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S, gate=gate,
                   raw_qk=raw, raw_beta=raw, raw_gate=raw)
    torch.cuda.synchronize()
    tol_o = TOL_F32 if dtype == torch.float32 else TOL_BF16_O
    assert_close(o, o_ref, tol_o, "decode T=%d o" % T)
    assert_close(S, s_ref, TOL_F32, "decode T=%d state" % T)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("B,H", [(3, 2), (40, 4)])
def test_multi_token_decode_head_shapes(dk, dv, B, H):
    """Every head shape, with few heads (16-column slices) and with enough
    heads for the wide slices."""
    T = 6
    inp = _inputs(B, T, H, dk, dv, torch.bfloat16, "channel", False, seed=7 + dk + dv + B,
                  init_std=None)
    S0 = decode_state(B, H, dk, dv, std=0.05, seed=B + dv)
    inp["init_state"] = S0
    o_ref, s_ref = _oracle(inp, "channel", False, clamp=False)
    g = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    S = S0.cuda()
    o = kda.decode(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S)
    torch.cuda.synchronize()
    assert_close(o, o_ref, TOL_BF16_O, "decode head shape o")
    assert_close(S, s_ref, TOL_F32, "decode head shape state")


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_multi_token_decode_full_gate_inside_a_chunk(gate):
    """log_alpha = -inf at the third of seven tokens clears the state there
    (a decay of exactly zero inside a call)."""
    B, T, H, d = 2, 7, 3, 128
    inp = _inputs(B, T, H, d, d, torch.float32, gate, False, seed=91, init_std=None)
    inp["log_alpha"][:, 2] = -float("inf")
    S0 = decode_state(B, H, d, d, std=0.05, seed=9)
    inp["init_state"] = S0
    o_ref, s_ref = _oracle(inp, gate, False, clamp=False)
    g = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    S = S0.cuda()
    o = kda.decode(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S, gate=gate)
    torch.cuda.synchronize()
    assert_close(o, o_ref, TOL_F32, "decode full gate o")
    assert_close(S, s_ref, TOL_F32, "decode full gate state")


@pytest.mark.parametrize("T", [2, 7, 16])
def test_multi_token_decode_equals_successive_steps(T):
    """One call over T tokens = T single-token calls, bit for bit (the same
    per-token arithmetic; the state stays in registers instead of HBM)."""
    B, H, d = 4, 8, 128
    inp = _inputs(B, T, H, d, d, torch.bfloat16, "channel", False, seed=61, init_std=None)
    g = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    S0 = decode_state(B, H, d, d, std=0.05, seed=61).cuda()
    S1 = S0.clone()
    o1 = kda.decode(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S1)
    S2 = S0.clone()
    o2 = torch.stack([kda.decode_step(*(g[n][:, t].contiguous() for n in
                                        ("q", "k", "v", "log_alpha", "beta")), S2)
                      for t in range(T)], 1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_decode_rejects_too_many_tokens():
    B, T, H, d = 1, kda.DECODE_MAX_TOKENS + 1, 1, 128
    x = torch.zeros(B, T, H, d, dtype=torch.bfloat16, device="cuda")
    la = torch.zeros(B, T, H, d, device="cuda")
    b = torch.zeros(B, T, H, device="cuda")
    S = torch.zeros(B, H, d, d, device="cuda")
    with pytest.raises(kda.KdaError) as e:
        kda.decode(x, x, x, la, b, S)
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED
