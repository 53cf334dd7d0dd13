"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle,
element by element on seeded inputs.

Tolerances (normwise max|x - ref| / max|ref|): fp32-input path 1e-4 for o and
the state; bf16-input path 1e-2 for o and 5e-3 for the final state.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import (decode_inputs, decode_state, prefill_inputs,
                                             varlen_lengths)
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, TOL_F32, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _to(inp, device=DEV):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _oracle(inp, log_alpha_min=None):
    """fp64 oracle on the same inputs. The chunked kernel is specified to
    apply the gate clamped at kda.CHUNK_LOG_ALPHA_MIN; its reference is the
    oracle on the clamped gate (identical whenever no gate is below it)."""
    lengths_cu = inp.get("cu_seqlens")
    cu = None if lengths_cu is None else lengths_cu.cpu().numpy().astype(np.int64)
    la = inp["log_alpha"].double()
    if log_alpha_min is not None:
        la = la.clamp(min=log_alpha_min)
    if cu is not None:
        q, k, v, b = (inp[n][0] for n in ("q", "k", "v", "beta"))
        return oracle.kda_forward(q, k, v, la[0], b, init_state=inp["init_state"], cu_seqlens=cu)
    return oracle.kda_forward(inp["q"], inp["k"], inp["v"], la, inp["beta"],
                              init_state=inp["init_state"])


def _gpu_prefill(inp, chunk):
    g = _to(inp)
    o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                       init_state=g["init_state"], cu_seqlens=g["cu_seqlens"], chunk=chunk)
    torch.cuda.synchronize()
    return o, s


def _check_prefill(inp, chunk, bf16=True):
    clamp = kda.CHUNK_LOG_ALPHA_MIN if (chunk == 64 and bf16) else None
    o_ref, s_ref = _oracle(inp, clamp)
    o, s = _gpu_prefill(inp, chunk)
    o = o[0] if inp.get("cu_seqlens") is not None else o
    if bf16:
        eo = assert_close(o, o_ref, TOL_BF16_O, "o")
        es = assert_close(s, s_ref, TOL_BF16_STATE, "final state")
    else:
        eo = assert_close(o, o_ref, TOL_F32, "o")
        es = assert_close(s, s_ref, TOL_F32, "final state")
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)
    return eo, es


# ---------------------------------------------------------------------------
# Tiny fp32 workload: B=1, H=1, T=256, dk=dv=64, zero initial state
# ---------------------------------------------------------------------------

def test_tiny_fp32_prefill():
    inp = prefill_inputs(1, 256, 1, 64, 64, dtype=torch.float32, seed=0)
    _check_prefill(inp, chunk=64, bf16=False)   # fp32 always runs the recurrent kernel


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 37, 130])
def test_recurrent_fp32_shapes(dk, dv, T):
    inp = prefill_inputs(2, T, 3, dk, dv, dtype=torch.float32, seed=T + dk, init_std=0.1)
    _check_prefill(inp, chunk=0, bf16=False)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)])
def test_recurrent_bf16(dk, dv):
    inp = prefill_inputs(2, 150, 2, dk, dv, dtype=torch.bfloat16, seed=3, init_std=0.1)
    _check_prefill(inp, chunk=0)


# ---------------------------------------------------------------------------
# Chunked tensor-core prefill (C = 64, dk = dv = 128, bf16)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 15, 16, 63, 64, 65, 128, 200, 333])
def test_chunk_prefill_lengths(T):
    inp = prefill_inputs(2, T, 3, 128, 128, dtype=torch.bfloat16, seed=T, init_std=0.1)
    _check_prefill(inp, chunk=64)


def test_chunk_prefill_zero_initial_state():
    inp = prefill_inputs(1, 257, 4, 128, 128, dtype=torch.bfloat16, seed=11)
    _check_prefill(inp, chunk=64)


def test_chunk_prefill_long_chain():
    inp = prefill_inputs(1, 2048, 2, 128, 128, dtype=torch.bfloat16, seed=5, init_std=0.1)
    _check_prefill(inp, chunk=64)


@pytest.mark.parametrize("gate", [0.0, -1e-6, -0.5, -5.0, -60.0, -np.inf])
@pytest.mark.parametrize("beta", [0.0, 1.0, None])
def test_chunk_gate_and_beta_extremes(gate, beta):
    inp = prefill_inputs(1, 150, 2, 128, 128, dtype=torch.bfloat16, seed=21, init_std=0.1)
    inp["log_alpha"].fill_(gate)
    if beta is not None:
        inp["beta"].fill_(beta)
    _check_prefill(inp, chunk=64)


@pytest.mark.parametrize("gate", [-60.0, -np.inf])
def test_chunk_clamped_gate_is_close_to_a_clear(gate):
    """A full clear (log_alpha far below the clamp) differs from the chunked
    kernel's clamped decay (alpha = e^-10) only at the 1e-4 level."""
    inp = prefill_inputs(1, 150, 2, 128, 128, dtype=torch.bfloat16, seed=23, init_std=1.0)
    inp["log_alpha"].fill_(gate)
    o_ref, s_ref = _oracle(inp)
    o, s = _gpu_prefill(inp, 64)
    assert_close(o, o_ref, TOL_BF16_O, "o")
    assert_close(s, s_ref, TOL_BF16_STATE, "final state")


@pytest.mark.parametrize("B,T,H", [(2, 333, 3), (1, 200, 40), (1, 130, 80)])
def test_chunk_strong_gates_against_the_unclamped_oracle(B, T, H):
    """Per-token, per-channel gates drawn uniformly in [-30, 0] straddle the
    chunked kernel's clamp at -10; its result stays within the bf16
    tolerances of the EXACT (unclamped) oracle. Shapes cover a ring of two
    CTAs (6 chains), two CTAs (40 chains) and one CTA per chain (80 chains)."""
    inp = prefill_inputs(B, T, H, 128, 128, dtype=torch.bfloat16, seed=41 + H, init_std=0.1)
    g = torch.Generator().manual_seed(1234 + H)
    inp["log_alpha"] = (-30.0 * torch.rand(inp["log_alpha"].shape, generator=g,
                                           dtype=torch.float64)).float()
    o_ref, s_ref = _oracle(inp)            # no clamp
    o, s = _gpu_prefill(inp, 64)
    assert_close(o, o_ref, TOL_BF16_O, "o vs unclamped oracle")
    assert_close(s, s_ref, TOL_BF16_STATE, "final state vs unclamped oracle")


@pytest.mark.parametrize("gate", [-5.0, -60.0, -np.inf])
def test_recurrent_applies_the_gate_exactly(gate):
    inp = prefill_inputs(1, 40, 2, 128, 128, dtype=torch.float32, seed=22, init_std=1.0)
    inp["log_alpha"].fill_(gate)
    _check_prefill(inp, chunk=0, bf16=False)


@pytest.mark.parametrize("gate", [-60.0, -np.inf])
def test_decode_clears_with_a_full_gate(gate):
    B, H, d = 3, 2, 128
    S = decode_state(B, H, d, d, std=1.0, seed=2).to(DEV)
    inp = _to(decode_inputs(B, H, d, d, dtype=torch.float32, seed=2))
    inp["log_alpha"].fill_(gate)
    kda.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S)
    expect = inp["beta"][..., None, None] * inp["k"][..., :, None] * inp["v"][..., None, :]
    torch.cuda.synchronize()
    assert_close(S, expect, TOL_F32, "cleared state")


def test_chunk_matches_recurrent_kernel():
    inp = prefill_inputs(2, 700, 2, 128, 128, dtype=torch.bfloat16, seed=8, init_std=0.1)
    o1, s1 = _gpu_prefill(inp, 64)
    o0, s0 = _gpu_prefill(inp, 0)
    assert_close(o1, o0, TOL_BF16_O, "chunk vs recurrent o")
    assert_close(s1, s0, TOL_BF16_STATE, "chunk vs recurrent state")


def test_final_state_may_alias_initial_state():
    inp = _to(prefill_inputs(2, 100, 2, 128, 128, dtype=torch.bfloat16, seed=4, init_std=0.1))
    ref_o, ref_s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               init_state=inp["init_state"].clone(), chunk=64)
    s = inp["init_state"].clone()
    o, s_out = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           init_state=s, final_state=s, chunk=64)
    torch.cuda.synchronize()
    assert s_out.data_ptr() == s.data_ptr()
    assert torch.equal(o, ref_o) and torch.equal(s, ref_s)


@pytest.mark.parametrize("split", [64, 100, 1])
@pytest.mark.parametrize("chunk", [64, 0])
def test_split_prefill_equals_whole(split, chunk):
    """Resume: prefill(T1) then prefill(T2) from its final state = prefill(T1 + T2)."""
    inp = _to(prefill_inputs(1, 260, 2, 128, 128, dtype=torch.bfloat16, seed=9, init_std=0.1))
    f = lambda sl, s0: kda.prefill(inp["q"][:, sl].contiguous(), inp["k"][:, sl].contiguous(),
                                   inp["v"][:, sl].contiguous(),
                                   inp["log_alpha"][:, sl].contiguous(),
                                   inp["beta"][:, sl].contiguous(), init_state=s0, chunk=chunk)
    o, s = f(slice(None), inp["init_state"])
    o1, s1 = f(slice(0, split), inp["init_state"])
    o2, s2 = f(slice(split, None), s1)
    assert_close(torch.cat([o1, o2], 1), o, TOL_BF16_O, "split o")
    assert_close(s2, s, TOL_BF16_STATE, "split state")


def test_non_default_stream():
    inp = prefill_inputs(1, 130, 2, 128, 128, dtype=torch.bfloat16, seed=12, init_std=0.1)
    o_ref, s_ref = _oracle(inp)
    g = _to(inp)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                           init_state=g["init_state"], chunk=64)
    st.synchronize()
    assert_close(o, o_ref, TOL_BF16_O, "o")
    assert_close(s, s_ref, TOL_BF16_STATE, "state")


# ---------------------------------------------------------------------------
# Packed variable-length sequences (cu_seqlens)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [64, 0])
def test_varlen_ragged(chunk):
    lengths = [0, 1, 63, 64, 65, 200, 300, 17]
    inp = prefill_inputs(1, 0, 2, 128, 128, dtype=torch.bfloat16, seed=13, init_std=0.1,
                         lengths=lengths)
    _check_prefill(inp, chunk=chunk)


def test_varlen_equals_separate_calls():
    lengths = [70, 5, 129]
    inp = _to(prefill_inputs(1, 0, 2, 128, 128, dtype=torch.bfloat16, seed=14, init_std=0.1,
                             lengths=lengths))
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], chunk=64)
    cu = inp["cu_seqlens"].tolist()
    for i in range(len(lengths)):
        sl = slice(cu[i], cu[i + 1])
        oi, si = kda.prefill(*(inp[n][:, sl].contiguous() for n in
                               ("q", "k", "v", "log_alpha", "beta")),
                             init_state=inp["init_state"][i:i + 1].contiguous(), chunk=64)
        assert torch.equal(o[:, sl], oi)
        assert torch.equal(s[i:i + 1], si)


# ---------------------------------------------------------------------------
# Decode step
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_decode_steps(dtype, dk, dv):
    B, H = 5, 3
    S = decode_state(B, H, dk, dv, std=0.05, seed=1)
    S_ref = S.double().numpy()
    S_gpu = S.to(DEV)
    for step in range(3):
        inp = decode_inputs(B, H, dk, dv, dtype=dtype, seed=1, step=step)
        o_ref, S_ref = oracle.kda_decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                              inp["beta"], S_ref)
        g = _to(inp)
        o = kda.decode_step(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S_gpu)
        torch.cuda.synchronize()
        tol_o = TOL_F32 if dtype == torch.float32 else TOL_BF16_O
        assert_close(o, o_ref, tol_o, "decode o step %d" % step)
        assert_close(S_gpu, S_ref, TOL_F32, "decode state step %d" % step)


def test_decode_graph_replay_matches_eager_and_oracle():
    """Decode steps captured once in a CUDA graph (how a single-sequence decode
    loop amortises launch latency) give the same bits as eager launches, and
    the oracle's values."""
    B, H, d, n = 1, 32, 128, 6
    S0 = decode_state(B, H, d, d, std=0.05, seed=21)
    ins = [_to(decode_inputs(B, H, d, d, dtype=torch.bfloat16, seed=21, step=i))
           for i in range(n)]
    names = ("q", "k", "v", "log_alpha", "beta")
    S_eager = S0.to(DEV)
    o_eager = [kda.decode_step(*(g[x] for x in names), S_eager) for g in ins]
    S_graph = S0.to(DEV)
    o_graph = torch.empty(n, B, H, d, dtype=torch.bfloat16, device=DEV)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap):
        for i, g in enumerate(ins):
            kda.decode_step(*(g[x] for x in names), S_graph, o=o_graph[i], stream=cap)
    torch.cuda.current_stream().wait_stream(cap)
    S_graph.copy_(S0.to(DEV))     # capture does not run the kernels; start from S0
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(S_graph, S_eager)
    for i in range(n):
        assert torch.equal(o_graph[i], o_eager[i])
    S_ref = S0.double().numpy()
    for i in range(n):
        o_ref, S_ref = oracle.kda_decode_step(*(ins[i][x].cpu() for x in names), S_ref)
        assert_close(o_graph[i], o_ref, TOL_BF16_O, "graph decode o step %d" % i)
    assert_close(S_graph, S_ref, TOL_F32, "graph decode state")
    del graph


def test_prefill_then_decode_equals_longer_prefill():
    inp = _to(prefill_inputs(2, 129, 2, 128, 128, dtype=torch.bfloat16, seed=15, init_std=0.1))
    o_all, s_all = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               init_state=inp["init_state"], chunk=0)
    sl = slice(0, 128)
    o_pre, s = kda.prefill(*(inp[n][:, sl].contiguous() for n in
                             ("q", "k", "v", "log_alpha", "beta")),
                           init_state=inp["init_state"], chunk=64)
    o_dec = kda.decode_step(*(inp[n][:, 128].contiguous() for n in
                              ("q", "k", "v", "log_alpha", "beta")), s)
    assert_close(o_dec, o_all[:, 128], TOL_BF16_O, "decode after prefill")
    assert_close(s, s_all, TOL_BF16_STATE, "state after decode")


def test_device_status_clean():
    st, detail = kda.device_status(reset=True)
    assert st == kda.KDA_OK and detail == 0
