"""GPU parity of the backward pass (kda_backward, through the C ABI) against
the fp64 oracle's reverse mode: every gradient of L = sum(o * Wo) +
sum(S_final * Ws) for random fixed weights Wo, Ws.

Tolerance (normwise max|x - ref| / max|ref| per gradient): 1e-4 for fp32
inputs (fp32 state and arithmetic, as the forward's fp32 path); for bf16
inputs the kernel and the oracle see the same bf16-rounded inputs and the
arithmetic is fp32, so the same 1e-4 applies except that d_o is bf16.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from tests.parity import TOL_F32, assert_close

pytestmark = pytest.mark.gpu


def _case(B, T, H, dk, dv, dtype, gate, seed, lengths=None):
    g = torch.Generator().manual_seed(seed)
    rn = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    n_seq = B if lengths is None else len(lengths)
    if lengths is not None:
        T = int(sum(lengths))
    q, k = rn(B, T, H, dk), rn(B, T, H, dk)
    q, k = q / q.norm(dim=-1, keepdim=True), k / k.norm(dim=-1, keepdim=True)
    gshape = {"channel": (B, T, H, dk), "scalar": (B, T, H), "none": None}[gate]
    la = None if gshape is None else torch.nn.functional.logsigmoid(rn(*gshape) + 3.0).float()
    inp = dict(q=q.to(dtype), k=k.to(dtype), v=rn(B, T, H, dv).to(dtype), log_alpha=la,
               beta=torch.sigmoid(rn(B, T, H)).float(),
               init_state=(rn(n_seq, H, dk, dv) * 0.1).float(),
               d_o=rn(B, T, H, dv).to(dtype), d_final=rn(n_seq, H, dk, dv).float(),
               cu_seqlens=None)
    if lengths is not None:
        inp["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                                         dtype=torch.int32)
    return inp


def _oracle(inp, gate):
    la = oracle.expand_gate(inp["log_alpha"], gate, inp["q"].shape[:-1], inp["q"].shape[-1])
    cu = inp["cu_seqlens"]
    names = ("q", "k", "v", "beta", "d_o")
    if cu is not None:
        q, k, v, b, do = (inp[n][0] for n in names)
        la = la[0]
        cu = cu.numpy().astype(np.int64)
    else:
        q, k, v, b, do = (inp[n] for n in names)
    g = oracle.kda_backward(q, k, v, la, b, do, init_state=inp["init_state"],
                            d_final=inp["d_final"], cu_seqlens=cu)
    if gate == "scalar":
        g["dlog_alpha"] = g["dlog_alpha"].sum(-1)
    if cu is not None:
        for n in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
            g[n] = g[n][None]
    return g


def _gpu(inp, gate):
    c = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    out = kda.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["d_o"],
                       init_state=c["init_state"], cu_seqlens=c["cu_seqlens"],
                       d_final=c["d_final"], gate=gate)
    torch.cuda.synchronize()
    return out


def _check(inp, gate, tol=TOL_F32):
    ref = _oracle(inp, gate)
    out = _gpu(inp, gate)
    for n in ("dq", "dk", "dv", "dbeta", "d_init") + (("dlog_alpha",) if gate != "none" else ()):
        assert_close(out[n], ref[n], tol, "backward %s (gate %s)" % (n, gate))


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
def test_backward_fp32(gate, dk, dv):
    _check(_case(2, 53, 2, dk, dv, torch.float32, gate, seed=dk + dv), gate)


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_backward_bf16_inputs(gate):
    _check(_case(1, 100, 3, 128, 128, torch.bfloat16, gate, seed=3), gate)


def test_backward_packed_sequences():
    inp = _case(1, 0, 2, 128, 128, torch.float32, "channel", seed=9,
                lengths=[0, 1, 15, 16, 17, 40, 3])
    _check(inp, "channel")


def test_backward_long_sequence_many_blocks():
    _check(_case(1, 700, 2, 128, 128, torch.float32, "channel", seed=11), "channel")


def test_backward_many_chains_wide_slices():
    # enough chains that each CTA takes 32 value columns (few chains take 8)
    _check(_case(2, 40, 80, 128, 128, torch.float32, "channel", seed=13), "channel")


def _raw_case(B, T, H, d, dtype, gate, seed, lengths=None):
    """The same case with raw projections: q, k ~ N(0, 1) unnormalised, beta
    logits ~ N(0, 1), gate logits ~ N(3, 1) (decays sigmoid(x) near 0.95)."""
    inp = _case(B, T, H, d, d, dtype, gate, seed, lengths=lengths)
    g = torch.Generator().manual_seed(seed + 1)
    shape = inp["q"].shape
    inp["q"] = torch.randn(shape, generator=g).to(dtype)
    inp["k"] = torch.randn(shape, generator=g).to(dtype)
    inp["beta"] = torch.randn(inp["beta"].shape, generator=g)
    if inp["log_alpha"] is not None:
        inp["log_alpha"] = torch.randn(inp["log_alpha"].shape, generator=g) + 3.0
    return inp


def _check_raw(inp, gate, tol=TOL_F32):
    cu = inp["cu_seqlens"]
    names = ("q", "k", "v", "log_alpha", "beta", "d_o")
    if cu is not None:
        args = [None if inp[n] is None else inp[n][0] for n in names]
        cu = cu.numpy().astype(np.int64)
    else:
        args = [inp[n] for n in names]
    ref = oracle.kda_backward_ex(*args, init_state=inp["init_state"], d_final=inp["d_final"],
                                 cu_seqlens=cu, gate=gate, raw_qk=True, raw_beta=True,
                                 raw_gate=True)
    c = {n: (x.cuda() if isinstance(x, torch.Tensor) else x) for n, x in inp.items()}
    out = kda.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["d_o"],
                       init_state=c["init_state"], cu_seqlens=c["cu_seqlens"],
                       d_final=c["d_final"], gate=gate, raw_qk=True, raw_beta=True,
                       raw_gate=True)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dbeta", "d_init") + (("dlog_alpha",) if gate != "none" else ()):
        r = ref[n][None] if cu is not None and n != "d_init" else ref[n]
        assert_close(out[n], r, tol, "backward through the prologue %s (gate %s)" % (n, gate))


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_through_the_prologue(gate, dtype):
    """Raw projections (SiLU + L2 normalisation of q and k, beta and gate
    logits): kda_backward_ex against the oracle's reverse mode through the
    same prologue."""
    _check_raw(_raw_case(2, 45, 3, 128, dtype, gate, seed=21 + len(gate)), gate)


def test_backward_through_the_prologue_packed_and_small_heads():
    _check_raw(_raw_case(1, 0, 2, 64, torch.float32, "channel", seed=23,
                         lengths=[5, 0, 33, 17]), "channel")
