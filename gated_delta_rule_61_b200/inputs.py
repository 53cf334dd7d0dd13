"""Seeded synthetic inputs for the KDA recurrence.

This module holds only the input recipe; none of the recurrence's arithmetic
lives here, and it imports neither the CUDA library nor the oracle, so both
sides (and the benchmark) can draw the same data from it.

Recipe (the pages name no dataset; these are the synthetic workloads):
  * q, k ~ N(0, 1), then L2-normalised over the head dimension per (token,
    head). The pages' DeltaNet layer normalises q and k before the recurrence
    ("DeltaNet, or Fast Weight Programmers" section of "22580: from GPT-2 to
    Kimi K3, explained"); the library takes them as given.
  * v ~ N(0, 1).
  * gate: log_alpha = log(sigmoid(x)), x ~ N(3, 1), one value per (token, head,
    key channel), computed in the generator's float type, stored as fp32.
  * beta = sigmoid(y), y ~ N(0, 1), one per (token, head), fp32 (the pages'
    per-token write strength is a sigmoid).
  * initial state ~ N(0, init_std^2) fp32 when init_std is given, else None.
  * q, k, v are rounded to the storage dtype (bf16 or fp32) here, so every
    consumer sees the same rounded values.
Draw order from one generator seeded with ``seed``: q, k, v, x, y, state.
Variable sequence lengths come from a separate numpy stream seeded with
(seed, 7): L_i = round(exp(U(ln lo, ln hi))).
On the CPU the draws are made in fp64; on a GPU in fp32 (the large workloads
do not fit fp64 temporaries). The two devices give different streams.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _float_type(device):
    return torch.float64 if torch.device(device).type == "cpu" else torch.float32


def _unit_rows(x):
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def varlen_lengths(n_seq: int, lo: int, hi: int, seed: int = 0) -> list[int]:
    """Log-uniform sequence lengths in [lo, hi] (inclusive after rounding)."""
    rng = np.random.default_rng([int(seed), 7])
    u = rng.uniform(math.log(lo), math.log(hi), size=n_seq)
    return [int(min(hi, max(lo, round(math.exp(x))))) for x in u]


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return torch.from_numpy(cu.astype(np.int32))


def prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, *,
                   dtype=torch.bfloat16, seed: int = 0, init_std=None,
                   device="cpu", lengths=None, gate_mean: float = 3.0):
    """Inputs for one prefill call.

    Dense batch: q, k, log_alpha [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    init_state [B, H, dk, dv] or None; cu_seqlens None.
    Packed varlen (``lengths`` given): B must be 1, T = sum(lengths), the
    tensors are [1, T, H, d], init_state is [len(lengths), H, dk, dv] and
    cu_seqlens is int32 [len(lengths) + 1] (on ``device``).
    """
    if lengths is not None:
        if B != 1:
            raise ValueError("packed sequences use B = 1")
        T = int(sum(lengths))
        n_seq = len(lengths)
    else:
        n_seq = B
    g = _gen(device, seed)
    ft = _float_type(device)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=ft)

    q = _unit_rows(randn(B, T, H, dk)).to(dtype)
    k = _unit_rows(randn(B, T, H, dk)).to(dtype)
    v = randn(B, T, H, dv).to(dtype)
    x = randn(B, T, H, dk).add_(gate_mean)
    log_alpha = torch.nn.functional.logsigmoid(x).to(torch.float32)
    del x
    y = randn(B, T, H)
    beta = torch.sigmoid(y).to(torch.float32)
    init_state = None
    if init_std is not None:
        init_state = (randn(n_seq, H, dk, dv) * float(init_std)).to(torch.float32)
    cu = None
    if lengths is not None:
        cu = cu_from_lengths(lengths).to(device)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                log_alpha=log_alpha.contiguous(), beta=beta.contiguous(),
                init_state=init_state, cu_seqlens=cu)


def decode_inputs(B: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                  seed: int = 0, step: int = 0, device="cpu",
                  gate_mean: float = 3.0):
    """Inputs of one decode step (one token per sequence): q, k, log_alpha
    [B, H, dk]; v [B, H, dv]; beta [B, H]. Seeded by (seed, step)."""
    g = _gen(device, int(seed) * 1000003 + int(step) + 1)
    ft = _float_type(device)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=ft)

    q = _unit_rows(randn(B, H, dk)).to(dtype)
    k = _unit_rows(randn(B, H, dk)).to(dtype)
    v = randn(B, H, dv).to(dtype)
    log_alpha = torch.nn.functional.logsigmoid(randn(B, H, dk).add_(gate_mean)).to(torch.float32)
    beta = torch.sigmoid(randn(B, H)).to(torch.float32)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                log_alpha=log_alpha.contiguous(), beta=beta.contiguous())


def decode_state(B: int, H: int, dk: int, dv: int, *, std: float = 0.05,
                 seed: int = 0, device="cpu"):
    """Initial decode cache [B, H, dk, dv] fp32 ~ N(0, std^2)."""
    g = _gen(device, int(seed) + 99991)
    ft = _float_type(device)
    s = torch.randn(B, H, dk, dv, generator=g, device=device, dtype=ft)
    return (s * float(std)).to(torch.float32).contiguous()
