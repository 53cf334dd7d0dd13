"""kda_prefill_noalloc: the packed variable-length chunked prefill for callers
that cannot allocate device memory (a plugin or hook that owns no allocator,
a runtime whose device memory is already reserved by its own pool, a
latency-critical path that must not allocate). Its scratch (the longest-first
sequence order) is a fixed array inside libkda.so instead of a caller
workspace, shared by every call on a device.

The GPU test calls it through the C ABI twice in a row, on different packed
inputs, and checks each result against kda_prefill (which takes a caller
workspace) within the bf16 tolerances of the parity tests. It runs last so a
failure here does not hide the other tests, and it must pass both alone in a
fresh process (where its first call performs the one-time device set-up) and
after the other tests.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import prefill_inputs
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, assert_close

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "kda.h")

FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: the size check fails first


def test_noalloc_rejects_too_many_sequences():
    n = kda.NOALLOC_MAX_SEQS + 1
    st = kda.lib().kda_prefill_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, n, 64, 2,
                                       FAKE, None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED


def test_binding_limits_match_the_header():
    text = open(HEADER).read()
    n = int(re.search(r"#define\s+KDA_NOALLOC_MAX_SEQS\s+(\d+)", text).group(1))
    clamp = float(re.search(r"#define\s+KDA_CHUNK_LOG_ALPHA_MIN\s+\(([-0-9.]+)f\)",
                            text).group(1))
    assert kda.NOALLOC_MAX_SEQS == n
    assert kda.CHUNK_LOG_ALPHA_MIN == clamp


def test_noalloc_requires_cu_seqlens():
    st = kda.lib().kda_prefill_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2,
                                       FAKE, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_noalloc_rejects_misaligned_tensors():
    bad = ctypes.c_void_p(0x10008)
    st = kda.lib().kda_prefill_noalloc(FAKE, FAKE, FAKE, bad, FAKE, None, FAKE, 1, 64, 2,
                                       FAKE, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda")
    cases = [([70, 5, 0, 129, 300, 64], 2, 31), ([17, 256, 1, 65, 200], 3, 32)]
    for lengths, H, seed in cases:
        inp = prefill_inputs(1, 0, H, 128, 128, dtype=torch.bfloat16, seed=seed, init_std=0.1,
                             lengths=lengths, device="cpu")
        g = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        o_ref, s_ref = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                   init_state=g["init_state"], cu_seqlens=g["cu_seqlens"],
                                   chunk=64)
        o = torch.empty_like(o_ref)
        s = torch.empty_like(s_ref)
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated(dev)
        kda.prefill_noalloc(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                            g["cu_seqlens"], init_state=g["init_state"], o=o, final_state=s)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(dev) == before
        # the same kernel over the same chains in the same order: bit for bit
        assert torch.equal(o, o_ref), "noalloc o (%d sequences)" % len(lengths)
        assert torch.equal(s, s_ref), "noalloc final state (%d sequences)" % len(lengths)
    st, detail = kda.device_status()
    assert st == kda.KDA_OK, (st, detail)


@pytest.mark.gpu
def test_noalloc_against_the_oracle():
    """One packed call checked directly against the fp64 oracle (gate
    clamped as the chunked kernel specifies)."""
    lengths = [90, 0, 3, 200]
    inp = prefill_inputs(1, 0, 2, 128, 128, dtype=torch.bfloat16, seed=33, init_std=0.1,
                         lengths=lengths)
    o_ref, s_ref = oracle.kda_forward(
        inp["q"][0], inp["k"][0], inp["v"][0],
        inp["log_alpha"][0].double().clamp(min=kda.CHUNK_LOG_ALPHA_MIN), inp["beta"][0],
        init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"].numpy().astype(np.int64))
    g = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, s = kda.prefill_noalloc(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                               g["cu_seqlens"], init_state=g["init_state"])
    torch.cuda.synchronize()
    assert_close(o[0], o_ref, TOL_BF16_O, "noalloc o vs oracle")
    assert_close(s, s_ref, TOL_BF16_STATE, "noalloc state vs oracle")


@pytest.mark.gpu
def test_noalloc_many_sequences_identity_order():
    """More than 8192 packed sequences (most of length 0 or 1) take the
    identity work order instead of the longest-first one; the result still
    matches the workspace entry point."""
    rng = np.random.default_rng(5)
    lengths = [int(x) for x in rng.choice([0, 1, 1, 2, 70], size=9000)]
    inp = prefill_inputs(1, 0, 1, 128, 128, dtype=torch.bfloat16, seed=34, init_std=0.1,
                         lengths=lengths, device="cuda")
    o_ref, s_ref = kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"],
                               chunk=64)
    o, s = kda.prefill_noalloc(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               inp["cu_seqlens"], init_state=inp["init_state"])
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
