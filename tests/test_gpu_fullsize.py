"""Parity at the full workload sizes, in the launch configuration the
benchmark times, on outputs the oracle can compute one chain at a time.

Workloads: prefill B=4 H=16 T=8192 d=128 (chunk 64); decode B=256 H=32 d=128;
packed varlen 64 sequences log-uniform in [128, 32768] with H=32; long
prefill T=1,048,576 H=32 followed by decode steps. The large inputs are
drawn on the GPU by the seeded generator and the sampled slices are copied to
the host for the oracle. Tolerances as in test_gpu_parity (normwise).
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
CLAMP = kda.CHUNK_LOG_ALPHA_MIN


def _chain_oracle(q, k, v, la, b, s0):
    """One (sequence, head) chain: q, k, la [T, dk]; v [T, dv]; b [T]; s0 [dk, dv]."""
    o, s = oracle.kda_forward(q[:, None], k[:, None], v[:, None],
                              la.double().clamp(min=CLAMP)[:, None], b[:, None],
                              init_state=None if s0 is None else s0[None, None])
    return o[:, 0], s[0, 0]


def test_prefill_mid_full_size_sampled_chains():
    B, T, H, d = 4, 8192, 16, 128
    inp = prefill_inputs(B, T, H, d, d, dtype=torch.bfloat16, seed=0, init_std=0.1,
                         device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], chunk=64)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (1, 7), (3, 15)):
        sl = lambda x: x[b, :, h].cpu()
        o_ref, s_ref = _chain_oracle(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                     sl(inp["log_alpha"]), inp["beta"][b, :, h].cpu(),
                                     inp["init_state"][b, h].cpu())
        assert_close(o[b, :, h], o_ref, TOL_BF16_O, "o chain (%d,%d)" % (b, h))
        assert_close(s[b, h], s_ref, TOL_BF16_STATE, "state chain (%d,%d)" % (b, h))


def test_decode_full_size():
    B, H, d = 256, 32, 128
    S = decode_state(B, H, d, d, std=0.05, seed=3, device="cuda")
    S_host = S.cpu().double().numpy()
    heads = [(0, 0), (17, 5), (255, 31), (128, 16)]
    for step in range(4):
        inp = decode_inputs(B, H, d, d, dtype=torch.bfloat16, seed=3, step=step, device="cuda")
        o = kda.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S)
        torch.cuda.synchronize()
        if step == 0:   # every head on the first step
            o_ref, S_host = oracle.kda_decode_step(*(inp[n].cpu() for n in
                                                     ("q", "k", "v", "log_alpha", "beta")),
                                                   S_host)
            assert_close(o, o_ref, TOL_BF16_O, "decode o, all heads")
            assert_close(S, S_host, TOL_F32, "decode state, all heads")
        else:           # sampled heads afterwards, continuing from the host copy
            for b, h in heads:
                sub = lambda n: inp[n][b:b + 1, h:h + 1].cpu()
                o_ref, s_new = oracle.kda_decode_step(sub("q"), sub("k"), sub("v"),
                                                      sub("log_alpha"), sub("beta"),
                                                      S_host[b:b + 1, h:h + 1])
                S_host[b:b + 1, h:h + 1] = s_new
                assert_close(o[b, h], o_ref[0, 0], TOL_BF16_O, "decode o (%d,%d)" % (b, h))
                assert_close(S[b, h], s_new[0, 0], TOL_F32, "decode state (%d,%d)" % (b, h))


def test_varlen_full_size_sampled_sequences():
    lengths = varlen_lengths(64, 128, 32768, seed=0)
    H, d = 32, 128
    inp = prefill_inputs(1, 0, H, d, d, dtype=torch.bfloat16, seed=0, init_std=0.1,
                         lengths=lengths, device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], chunk=64)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    order = np.argsort(lengths)
    picks = [int(order[0]), int(order[len(order) // 2]), int(order[-1])]   # short, mid, longest
    for i in picks:
        h = (7 * i) % H
        a, e = cu[i], cu[i + 1]
        sl = lambda x: x[0, a:e, h].cpu()
        o_ref, s_ref = _chain_oracle(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                     sl(inp["log_alpha"]), inp["beta"][0, a:e, h].cpu(),
                                     inp["init_state"][i, h].cpu())
        assert_close(o[0, a:e, h], o_ref, TOL_BF16_O, "o seq %d (len %d)" % (i, e - a))
        assert_close(s[i, h], s_ref, TOL_BF16_STATE, "state seq %d (len %d)" % (i, e - a))


def test_long_context_prefill_then_decode():
    """T = 1,048,576, H = 32, zero initial state: the first 16384 tokens of
    sampled heads against the oracle; the whole sequence against a split
    prefill (at 524288 + 37) resumed from the first part's state; then decode
    steps from the final state, checked by the oracle started from the GPU's
    final state."""
    T, H, d, split = 1 << 20, 32, 128, (1 << 19) + 37
    inp = prefill_inputs(1, T, H, d, d, dtype=torch.bfloat16, seed=4, device="cuda")
    o, s = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], chunk=64)
    torch.cuda.synchronize()
    n0 = 16384
    for h in (0, 13, 31):
        sl = lambda x: x[0, :n0, h].cpu()
        o_ref, _ = _chain_oracle(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                 sl(inp["log_alpha"]), inp["beta"][0, :n0, h].cpu(), None)
        assert_close(o[0, :n0, h], o_ref, TOL_BF16_O, "o first %d tokens, head %d" % (n0, h))
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
