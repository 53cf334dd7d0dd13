"""Parity at the full workload sizes, in the launch configuration the
benchmark times.

Workloads: prefill B=4 H=16 T=8192 d=128 (chunk 64): every chain; decode
B=256 H=32 d=128 for 1000 in-place steps: every head's output at every step
and every head's state after the last step; packed varlen 64 sequences
log-uniform in [128, 32768] with H=32: every sequence on four heads; long
prefill T=1,048,576 H=32: the first 16384 tokens of every head, the whole
sequence against a split prefill, then decode steps; the prefill's other gate
forms and the fused prologue at its full size, every chain; 16-token decode
calls at the decode size; the backward at the prefill size. The large inputs are
drawn on the GPU by the seeded generator and copied to the host for the
oracle. Tolerances as in test_gpu_parity (normwise).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import (decode_inputs, decode_state, prefill_inputs,
                                             varlen_lengths)
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, TOL_F32, assert_close, normwise

pytestmark = pytest.mark.gpu
CLAMP = kda.CHUNK_LOG_ALPHA_MIN


def test_prefill_mid_full_size_every_chain():
    B, T, H, d = 4, 8192, 16, 128
    inp = prefill_inputs(B, T, H, d, d, dtype=torch.bfloat16, seed=0, init_std=0.1,
                         device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], chunk=64)
    torch.cuda.synchronize()
    host = {n: inp[n].cpu() for n in ("q", "k", "v", "log_alpha", "beta", "init_state")}
    o_ref, s_ref = oracle.kda_forward(host["q"], host["k"], host["v"],
                                      host["log_alpha"].double().clamp(min=CLAMP),
                                      host["beta"], init_state=host["init_state"])
    o_h, s_h = o.cpu(), s.cpu()
    worst_o = max(normwise(o_h[b, :, h], o_ref[b, :, h]) for b in range(B) for h in range(H))
    worst_s = max(normwise(s_h[b, h], s_ref[b, h]) for b in range(B) for h in range(H))
    assert worst_o <= TOL_BF16_O, "o, worst of 64 chains: %.3e" % worst_o
    assert worst_s <= TOL_BF16_STATE, "final state, worst of 64 chains: %.3e" % worst_s


def test_decode_full_size_1000_steps():
    """1000 in-place decode steps at B=256, H=32. The oracle runs each head's
    1000 steps as one token loop from the same initial state (a decode step is
    the recurrence with one token), in blocks of heads."""
    B, H, d, n_steps = 256, 32, 128, 1000
    S = decode_state(B, H, d, d, std=0.05, seed=3, device="cuda")
    S0 = S.cpu()
    names = ("q", "k", "v", "log_alpha", "beta")
    ins = {n: [] for n in names}
    outs = torch.empty(n_steps, B, H, d, dtype=torch.bfloat16, device="cuda")
    for step in range(n_steps):
        inp = decode_inputs(B, H, d, d, dtype=torch.bfloat16, seed=3, step=step, device="cuda")
        kda.decode_step(*(inp[n] for n in names), S, o=outs[step])
        for n in names:
            ins[n].append(inp[n])
    torch.cuda.synchronize()
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)
    # [steps, B * H, d] token-major layout: each head is a chain of 1000 tokens
    seq = {n: torch.stack(ins[n]).reshape(n_steps, B * H, -1) for n in ("q", "k", "v",
                                                                      "log_alpha")}
    seq["beta"] = torch.stack(ins["beta"]).reshape(n_steps, B * H)
    del ins
    outs = outs.reshape(n_steps, B * H, d)
    S_gpu = S.reshape(B * H, d, d).cpu()
    S0 = S0.reshape(B * H, d, d)
    worst_o = worst_s = 0.0
    blk = 512
    for h0 in range(0, B * H, blk):
        sl = slice(h0, h0 + blk)
        o_ref, s_ref = oracle.kda_forward(*(seq[n][:, sl].cpu() for n in names),
                                          init_state=S0[None, sl])
        o_blk = outs[:, sl].cpu().double().numpy()
        for step in range(n_steps):      # every head's output at every step
            worst_o = max(worst_o, normwise(o_blk[step], o_ref[step]))
        worst_s = max(worst_s, normwise(S_gpu[sl], s_ref[0]))
    assert worst_o <= TOL_BF16_O, "decode o, worst step: %.3e" % worst_o
    assert worst_s <= TOL_F32, "decode state after 1000 steps: %.3e" % worst_s


def test_varlen_full_size_every_sequence():
    lengths = varlen_lengths(64, 128, 32768, seed=0)
    H, d = 32, 128
    inp = prefill_inputs(1, 0, H, d, d, dtype=torch.bfloat16, seed=0, init_std=0.1,
                         lengths=lengths, device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], chunk=64)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    host = {n: inp[n][0].cpu() for n in ("q", "k", "v", "log_alpha", "beta")}
    o_h, s_h, s0 = o[0].cpu(), s.cpu(), inp["init_state"].cpu()
    cu64 = np.asarray(cu, dtype=np.int64)
    for off in (0, 11, 19, 30):
        # every sequence on head (7 i + off) mod H, as one packed call of
        # single-head chains (the oracle threads over them)
        heads = [(7 * i + off) % H for i in range(len(lengths))]
        pick = lambda x: torch.cat([x[cu[i]:cu[i + 1], heads[i]:heads[i] + 1]
                                    for i in range(len(lengths))])
        o_ref, s_ref = oracle.kda_forward(
            pick(host["q"]), pick(host["k"]), pick(host["v"]),
            pick(host["log_alpha"]).double().clamp(min=CLAMP), pick(host["beta"]),
            init_state=torch.stack([s0[i, h:h + 1] for i, h in enumerate(heads)]),
            cu_seqlens=cu64)
        o_gpu = pick(o_h)
        for i, h in enumerate(heads):
            a, e = cu[i], cu[i + 1]
            assert_close(o_gpu[a:e, 0], o_ref[a:e, 0], TOL_BF16_O,
                         "o seq %d head %d (len %d)" % (i, h, e - a))
            assert_close(s_h[i, h], s_ref[i, 0], TOL_BF16_STATE,
                         "state seq %d head %d (len %d)" % (i, h, e - a))


def test_long_context_prefill_then_decode():
    """T = 1,048,576, H = 32, zero initial state: the first 16384 tokens of
    every head against the oracle; the whole sequence against a split
    prefill (at 524288 + 37) resumed from the first part's state; then decode
    steps from the final state, checked by the oracle started from the GPU's
    final state."""
    T, H, d, split = 1 << 20, 32, 128, (1 << 19) + 37
    inp = prefill_inputs(1, T, H, d, d, dtype=torch.bfloat16, seed=4, device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], chunk=64)
    torch.cuda.synchronize()
    n0 = 16384
    head = {n: inp[n][:, :n0].cpu() for n in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, _ = oracle.kda_forward(head["q"], head["k"], head["v"],
                                  head["log_alpha"].double().clamp(min=CLAMP), head["beta"])
    o_h = o[:, :n0].cpu()
    for h in range(H):
        assert_close(o_h[0, :, h], o_ref[0, :, h], TOL_BF16_O,
                     "o first %d tokens, head %d" % (n0, h))
    part = lambda x, a, e: x[:, a:e].contiguous()
    names = ("q", "k", "v", "log_alpha", "beta")
    o1, s1 = kda.prefill(*(part(inp[n], 0, split) for n in names), chunk=64)
    o2, s2 = kda.prefill(*(part(inp[n], split, T) for n in names), init_state=s1, chunk=64)
    torch.cuda.synchronize()
    assert_close(s2, s, TOL_BF16_STATE, "split-prefill final state")
    assert_close(o2[:, -4096:], o[:, -4096:], TOL_BF16_O, "split-prefill o (last 4096 tokens)")
    assert_close(o1[:, :4096], o[:, :4096], TOL_BF16_O, "split-prefill o (first 4096 tokens)")
    del o1, o2, inp
    torch.cuda.empty_cache()
    S_host = s.cpu().double().numpy()
    for step in range(8):
        dinp = decode_inputs(1, H, d, d, dtype=torch.bfloat16, seed=4, step=step, device="cuda")
        od = kda.decode_step(dinp["q"], dinp["k"], dinp["v"], dinp["log_alpha"], dinp["beta"], s)
        torch.cuda.synchronize()
        o_ref, S_host = oracle.kda_decode_step(*(dinp[n].cpu() for n in names), S_host)
        assert_close(od, o_ref, TOL_BF16_O, "long-context decode o step %d" % step)
        assert_close(s, S_host, TOL_F32, "long-context decode state step %d" % step)
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)


@pytest.mark.parametrize("form", ["scalar", "none", "raw"])
def test_prefill_forms_full_size_every_chain(form):
    """The other gate forms and the fused prologue at the benchmark's prefill
    size (B=4 T=8192 H=16, as the benchmark times them): every chain against
    the oracle. Scalar gate: log sigmoid(N(3, 1)) per (token, head); raw:
    unnormalised N(0, 1) q and k, beta logits N(0, 1) and gate logits N(3, 1)
    per key channel, the clamp applied to log sigmoid of the logits."""
    B, T, H, d = 4, 8192, 16, 128
    inp = prefill_inputs(B, T, H, d, d, dtype=torch.bfloat16, seed=5, init_std=0.1,
                         device="cuda")
    g = torch.Generator(device="cuda").manual_seed(55)
    gate, raw = {"scalar": ("scalar", False), "none": ("none", False),
                 "raw": ("channel", True)}[form]
    q, k, la, beta = inp["q"], inp["k"], inp["log_alpha"], inp["beta"]
    if form == "scalar":
        la = torch.nn.functional.logsigmoid(torch.randn(B, T, H, device="cuda", generator=g) + 3.0)
    elif form == "none":
        la = None
    else:
        q = torch.randn(q.shape, device="cuda", generator=g).to(torch.bfloat16)
        k = torch.randn(k.shape, device="cuda", generator=g).to(torch.bfloat16)
        beta = torch.randn(beta.shape, device="cuda", generator=g)
        la = torch.randn(la.shape, device="cuda", generator=g) + 3.0
    o, s = kda.prefill(q, k, inp["v"], la, beta, init_state=inp["init_state"], chunk=64,
                       gate=gate, raw_qk=raw, raw_beta=raw, raw_gate=raw)
    torch.cuda.synchronize()
    la_h = None
    if la is not None:
        la_h = la.cpu().double()
        if raw:
            la_h = torch.from_numpy(oracle.log_sigmoid(la_h))
        la_h = la_h.clamp(min=CLAMP)
    o_ref, s_ref = oracle.kda_forward_ex(q.cpu(), k.cpu(), inp["v"].cpu(), la_h, beta.cpu(),
                                         init_state=inp["init_state"].cpu(), gate=gate,
                                         raw_qk=raw, raw_beta=raw, raw_gate=False)
    o_h, s_h = o.cpu(), s.cpu()
    worst_o = max(normwise(o_h[b, :, h], o_ref[b, :, h]) for b in range(B) for h in range(H))
    worst_s = max(normwise(s_h[b, h], s_ref[b, h]) for b in range(B) for h in range(H))
    assert worst_o <= TOL_BF16_O, "%s: o, worst of 64 chains: %.3e" % (form, worst_o)
    assert worst_s <= TOL_BF16_STATE, "%s: final state, worst of 64 chains: %.3e" % (form, worst_s)


def test_multi_token_decode_full_size():
    """16 tokens per call at the benchmark's decode size (B=256 H=32 d=128,
    per-channel gate, bf16 inputs): every head's 16 outputs and final state
    against the oracle's token loop from the same cached state."""
    B, T, H, d = 256, 16, 32, 128
    g = torch.Generator(device="cuda").manual_seed(77)
    x = {n: torch.randn(B, T, H, d, device="cuda", generator=g) for n in ("q", "k", "v")}
    for n in ("q", "k"):
        x[n] = x[n] / x[n].norm(dim=-1, keepdim=True)
    x = {n: t.to(torch.bfloat16) for n, t in x.items()}
    la = torch.nn.functional.logsigmoid(torch.randn(B, T, H, d, device="cuda", generator=g) + 3.0)
    b = torch.sigmoid(torch.randn(B, T, H, device="cuda", generator=g))
    S = decode_state(B, H, d, d, std=0.05, seed=4, device="cuda")
    S0 = S.cpu()
    o = kda.decode(x["q"], x["k"], x["v"], la, b, S)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), la.cpu(), b.cpu(),
                                      init_state=S0)
    assert_close(o.cpu(), o_ref, TOL_BF16_O, "multi-token decode o, all heads")
    worst_s = max(normwise(S[bb].cpu(), s_ref[bb]) for bb in range(B))
    assert worst_s <= TOL_F32, "multi-token decode state, worst sequence: %.3e" % worst_s


def test_backward_full_size():
    """The backward at the benchmark's prefill size (B=4 T=8192 H=16, bf16,
    per-channel gate): every gradient against the oracle's fp64 reverse mode,
    per (sequence, head) for the state gradient."""
    B, T, H, d = 4, 8192, 16, 128
    inp = prefill_inputs(B, T, H, d, d, dtype=torch.bfloat16, seed=6, init_std=0.1,
                         device="cuda")
    g = torch.Generator(device="cuda").manual_seed(66)
    d_o = torch.randn(inp["v"].shape, device="cuda", generator=g).to(torch.bfloat16)
    d_fin = torch.randn(inp["init_state"].shape, device="cuda", generator=g)
    out = kda.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o,
                       init_state=inp["init_state"], d_final=d_fin)
    torch.cuda.synchronize()
    ref = oracle.kda_backward(inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu(),
                              inp["log_alpha"].cpu(), inp["beta"].cpu(), d_o.cpu(),
                              init_state=inp["init_state"].cpu(), d_final=d_fin.cpu())
    for n in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        assert_close(out[n].cpu(), ref[n], TOL_F32, "full-size backward %s" % n)
    worst = max(normwise(out["d_init"][b, h].cpu(), ref["d_init"][b, h])
                for b in range(B) for h in range(H))
    assert worst <= TOL_F32, "full-size backward d_init, worst chain: %.3e" % worst
