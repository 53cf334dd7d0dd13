"""Parity of the chunked prefill in each of its launch shapes.

The chunked kernel serves a (sequence, head) chain with one CTA, or, when
the final state is requested and chains are few, with a ring of two or four
CTAs (a thread-block cluster) that hand the state around. Which shape runs
depends only on the number of chains and on whether the final state is
requested (4 CTAs when 4 x chains fit on the GPU's SMs, else 2 when 2 x
chains fit, else 1), so these tests pick chain counts that land in each
shape on a 148-SM B200, with ragged lengths, single partial chunks, empty
packed sequences, and a chain count at each boundary. Every case is checked
against the fp64 oracle within the bf16 tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import prefill_inputs
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, assert_close

pytestmark = pytest.mark.gpu
CLAMP = kda.CHUNK_LOG_ALPHA_MIN


def _n_sm():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _ring_for(chains):
    n = _n_sm()
    return 4 if 4 * chains <= n else 2 if 2 * chains <= n else 1


def _oracle(inp):
    la = inp["log_alpha"].double().clamp(min=CLAMP)
    cu = inp.get("cu_seqlens")
    if cu is not None:
        q, k, v, b = (inp[n][0] for n in ("q", "k", "v", "beta"))
        return oracle.kda_forward(q, k, v, la[0], b, init_state=inp["init_state"],
                                  cu_seqlens=cu.numpy().astype(np.int64))
    return oracle.kda_forward(inp["q"], inp["k"], inp["v"], la, inp["beta"],
                              init_state=inp["init_state"])


def _run(inp, output_final_state=True):
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                       init_state=g["init_state"], cu_seqlens=g["cu_seqlens"], chunk=64,
                       output_final_state=output_final_state)
    torch.cuda.synchronize()
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)
    return o, s


@pytest.mark.parametrize("B,H,T", [
    (5, 10, 200),    # 50 chains: two CTAs per chain, 3 full chunks + 8 tokens
    (5, 10, 65),     # two chunks, the second one token long
    (5, 10, 64),     # one chunk: the second CTA of each ring has nothing to do
    (1, 74, 130),    # 74 chains: the largest count that still gets two CTAs
    (1, 37, 130),    # 37 chains: the largest count that still gets four CTAs
    (1, 38, 300),    # 38 chains: the smallest count that gets two CTAs
    (4, 20, 150),    # 80 chains: one CTA per chain
    (1, 75, 97),     # 75 chains: the smallest count that gets one CTA
])
def test_dense_batch_each_launch_shape(B, H, T):
    inp = prefill_inputs(B, T, H, 128, 128, dtype=torch.bfloat16, seed=B * 1000 + H + T,
                         init_std=0.1)
    o_ref, s_ref = _oracle(inp)
    o, s = _run(inp)
    ring = _ring_for(B * H)
    assert_close(o, o_ref, TOL_BF16_O, "o (ring of %d)" % ring)
    assert_close(s, s_ref, TOL_BF16_STATE, "final state (ring of %d)" % ring)


@pytest.mark.parametrize("B,H,T", [(2, 3, 333), (5, 10, 200)])
def test_without_final_state_one_cta_per_chain(B, H, T):
    """No final state requested: always one CTA per chain (no hand-over slot)."""
    inp = prefill_inputs(B, T, H, 128, 128, dtype=torch.bfloat16, seed=77 + T, init_std=0.1)
    o_ref, _ = _oracle(inp)
    o, s = _run(inp, output_final_state=False)
    assert s is None
    assert_close(o, o_ref, TOL_BF16_O, "o without final state")


@pytest.mark.parametrize("lengths,H", [
    ([0, 1, 63, 64, 65, 130, 200, 17], 5),    # 40 chains: two CTAs per chain
    ([40, 0, 129, 3, 64, 250, 1, 90, 66, 12], 10),   # 100 chains: one CTA per chain
])
def test_packed_sequences_each_launch_shape(lengths, H):
    inp = prefill_inputs(1, 0, H, 128, 128, dtype=torch.bfloat16, seed=len(lengths) * H,
                         init_std=0.1, lengths=lengths)
    o_ref, s_ref = _oracle(inp)
    o, s = _run(inp)
    ring = _ring_for(len(lengths) * H)
    assert_close(o[0], o_ref, TOL_BF16_O, "o (packed, ring of %d)" % ring)
    assert_close(s, s_ref, TOL_BF16_STATE, "final state (packed, ring of %d)" % ring)
    # an empty sequence passes its initial state through unchanged
    for i, n in enumerate(lengths):
        if n == 0:
            assert torch.equal(s[i].cpu(), inp["init_state"][i].float())


def test_launch_shape_does_not_change_the_bits():
    """Chains are independent and every shape runs the same per-chunk
    arithmetic (the state crosses L2 as exact fp32), so the same chains give
    the same bits whether they run with one CTA each (80 chains), in rings of
    two (40 chains) or in rings of four (6 chains)."""
    assert _ring_for(80) == 1 and _ring_for(40) == 2 and _ring_for(6) == 4
    inp = prefill_inputs(2, 150, 40, 128, 128, dtype=torch.bfloat16, seed=88, init_std=0.1,
                         device="cpu")
    o80, s80 = _run(inp)
    part = {n: (inp[n][:1].contiguous() if inp[n] is not None else None) for n in inp}
    o40, s40 = _run(part)
    part = {n: (inp[n][:, :, :3].contiguous() if n in ("q", "k", "v", "log_alpha", "beta")
                else inp[n]) for n in inp}
    part["init_state"] = inp["init_state"][:, :3].contiguous()
    o6, s6 = _run(part)
    assert torch.equal(o40, o80[:1]) and torch.equal(s40, s80[:1])
    assert torch.equal(o6, o80[:, :, :3]) and torch.equal(s6, s80[:, :3])
