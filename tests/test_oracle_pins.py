"""Pins for the fp64 CPU oracle: each test checks it against something other
than itself (an invariant the pages state, a closed form, an unrolled product
of matrices, an independently derived chunk algebra, hand-worked values).

Sources ("22580: from GPT-2 to Kimi K3, explained" = temp07.ru page, its
English original at marvinlee.cn, the wps.hkprog.org digest, the ai-flip.ru
KDA explainer):
  * no change when v_new equals v_old (digest, section "DeltaNet: now memory
    can be edited"; the aivibenews summary of the delta rule);
  * a unit key reads back exactly what was written, a repeated key is
    overwritten (temp07.ru, "DeltaNet, or Fast Weight Programmers");
  * alpha = 1 is the pure delta rule, alpha = 0 clears memory (temp07.ru,
    "Gated Delta Net");
  * one decay per key channel (temp07.ru "KDA / Kimi Linear"; ai-flip.ru,
    channel-wise gating as a diagonal gate matrix);
  * Householder transition form and chunk-wise parallel form (temp07.ru,
    "DeltaNet, or Parallelizing Linear Transformers with Delta Rule").
"""
import json
import os

import numpy as np
import pytest

import oracle
from tests import chunk_algebra as ca

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_case(rng, T, H, dk, dv, gate=True, beta_range=(0.0, 1.0)):
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    la = (np.log(1.0 / (1.0 + np.exp(-(rng.standard_normal((T, H, dk)) + 2.0))))
          if gate else np.zeros((T, H, dk)))
    b = rng.uniform(*beta_range, size=(T, H))
    return q, k, v, la, b


def _fwd(q, k, v, la, b, S0=None):
    """Single sequence, returns (o [T,H,dv], S [H,dk,dv])."""
    s0 = None if S0 is None else S0[None]
    o, fin = oracle.kda_forward(q, k, v, la, b, init_state=s0)
    return o, fin[0]


# ---------------------------------------------------------------------------
# Invariants stated in prose on the pages
# ---------------------------------------------------------------------------

def check_no_change(fwd, rng):
    """v_t equal to what the key reads from the decayed state => S_t = S'."""
    H, dk, dv = 2, 6, 5
    S0 = rng.standard_normal((H, dk, dv))
    q, k, _, la, b = _rand_case(rng, 1, H, dk, dv)
    Sd = np.exp(la[0])[:, :, None] * S0              # Diag(alpha) S0, per head
    v = np.einsum("hkv,hk->hv", Sd, k[0])[None]      # v_old at k
    o, S = fwd(q, k, v, la, b, S0)
    np.testing.assert_allclose(S, Sd, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o[0], np.einsum("hkv,hk->hv", Sd, q[0]), atol=1e-13)


def check_overwrite_retrieval(fwd, rng):
    """alpha = 1, beta = 1, orthonormal keys: each query at a written key
    returns exactly that key's value; a second write to a key replaces it."""
    dk, dv = 8, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T                                      # rows orthonormal
    vals = rng.standard_normal((dk, dv))
    new_v3 = rng.standard_normal(dv)
    # 8 writes, 1 overwrite of key 3, then 8 read-only steps (beta = 0).
    T = dk + 1 + dk
    k = np.zeros((T, 1, dk)); v = np.zeros((T, 1, dv)); q = np.zeros((T, 1, dk))
    b = np.zeros((T, 1)); la = np.zeros((T, 1, dk))
    k[:dk, 0] = keys; v[:dk, 0] = vals; b[:dk] = 1.0; q[:dk, 0] = keys
    k[dk, 0] = keys[3]; v[dk, 0] = new_v3; b[dk] = 1.0; q[dk, 0] = keys[3]
    for i in range(dk):
        t = dk + 1 + i
        k[t, 0] = keys[(i + 1) % dk]   # any key: beta = 0 makes it inert
        q[t, 0] = keys[i]
    o, _ = fwd(q, k, v, la, b)
    expect = vals.copy(); expect[3] = new_v3
    np.testing.assert_allclose(o[dk + 1:, 0], expect, atol=1e-12)
    # each write reads back its own value right away (read-out after write)
    np.testing.assert_allclose(o[:dk, 0], vals, atol=1e-12)
    np.testing.assert_allclose(o[dk, 0], new_v3, atol=1e-12)


def check_clear(fwd, rng):
    """log_alpha = -inf on every channel at step t => S_t = beta k v^T."""
    T, H, dk, dv = 7, 2, 5, 4
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv)
    S0 = rng.standard_normal((H, dk, dv))
    la[-1] = -np.inf
    o, S = fwd(q, k, v, la, b, S0)
    expect = b[-1][:, None, None] * k[-1][:, :, None] * v[-1][:, None, :]
    np.testing.assert_allclose(S, expect, atol=1e-14)


def check_channel_gate_rows(fwd, rng):
    """The gate acts per KEY channel (rows of the dk x dv state): with
    beta = 0 and log_alpha = -inf on a subset of channels, exactly those
    rows are zeroed and the others are untouched."""
    H, dk, dv = 1, 6, 4
    S0 = rng.standard_normal((H, dk, dv))
    q, k, v, la, b = _rand_case(rng, 1, H, dk, dv)
    b[:] = 0.0
    la[:] = 0.0
    la[0, 0, [1, 4]] = -np.inf
    _, S = fwd(q, k, v, la, b, S0)
    expect = S0.copy(); expect[:, [1, 4], :] = 0.0
    np.testing.assert_array_equal(S, expect)


def check_no_update(fwd, rng):
    """alpha = 1, beta = 0: the state never changes, o_t = S0^T q_t."""
    T, H, dk, dv = 5, 2, 4, 3
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv, gate=False)
    b[:] = 0.0
    S0 = rng.standard_normal((H, dk, dv))
    o, S = fwd(q, k, v, la, b, S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, np.einsum("hkv,thk->thv", S0, q), atol=1e-14)


def check_product_form(fwd, rng):
    """Unrolled product of dense transition matrices (Householder form with
    the diagonal gate): S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T."""
    for T, dk, dv in ((1, 3, 2), (4, 5, 3), (6, 6, 6), (6, 4, 5)):
        q, k, v, la, b = _rand_case(rng, T, 1, dk, dv)
        S0 = rng.standard_normal((1, dk, dv))
        o, S = fwd(q, k, v, la, b, S0)
        A = [(np.eye(dk) - b[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(la[t, 0]))
             for t in range(T)]
        for tt in range(1, T + 1):   # state after tt tokens, as a sum of products
            P = np.eye(dk)
            St = np.zeros((dk, dv))
            for t in range(tt - 1, -1, -1):
                St += P @ (b[t, 0] * np.outer(k[t, 0], v[t, 0]))
                P = P @ A[t]
            St += P @ S0[0]
            np.testing.assert_allclose(o[tt - 1, 0], St.T @ q[tt - 1, 0], atol=1e-12)
        np.testing.assert_allclose(S[0], St, atol=1e-12)


def check_resume(fwd, rng):
    """Running T1 tokens, then T2 more from the returned state, equals one
    run over T1 + T2 tokens, bit for bit (identical operation order)."""
    T1, T2, H, dk, dv = 9, 7, 2, 5, 4
    q, k, v, la, b = _rand_case(rng, T1 + T2, H, dk, dv)
    S0 = rng.standard_normal((H, dk, dv))
    o, S = fwd(q, k, v, la, b, S0)
    o1, S1 = fwd(q[:T1], k[:T1], v[:T1], la[:T1], b[:T1], S0)
    o2, S2 = fwd(q[T1:], k[T1:], v[T1:], la[T1:], b[T1:], S1)
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(S2, S)


PINS = [check_no_change, check_overwrite_retrieval, check_clear,
        check_channel_gate_rows, check_no_update, check_product_form,
        check_resume]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(_fwd, np.random.default_rng(1234))


# ---------------------------------------------------------------------------
# Independent algebra: chunked forms derived from the recurrence
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("C", [1, 4, 16])
def test_ungated_chunk_form_matches(C):
    rng = np.random.default_rng(7)
    T, dk, dv = 48, 8, 6
    q, k, v, _, b = _rand_case(rng, T, 1, dk, dv, gate=False)
    S0 = rng.standard_normal((dk, dv))
    O_ref, S_ref = _fwd(q, k, v, np.zeros((T, 1, dk)), b, S0[None])
    O, S = ca.chunk_delta_ungated(q[:, 0], k[:, 0], v[:, 0], b[:, 0], C, S0)
    np.testing.assert_allclose(O, O_ref[:, 0], atol=1e-11)
    np.testing.assert_allclose(S, S_ref[0], atol=1e-11)


@pytest.mark.parametrize("T,C,sub", [(64, 64, 16), (200, 64, 16), (131, 32, 8),
                                     (65, 64, 16), (1, 64, 16)])
def test_gated_chunk_form_matches(T, C, sub):
    rng = np.random.default_rng(T + C)
    dk, dv = 16, 12
    q, k, v, la, b = _rand_case(rng, T, 1, dk, dv)
    S0 = rng.standard_normal((dk, dv))
    O_ref, S_ref = _fwd(q, k, v, la, b, S0[None])
    O, S = ca.chunk_kda_gated(q[:, 0], k[:, 0], v[:, 0], la[:, 0], b[:, 0], C, S0, sub)
    np.testing.assert_allclose(O, O_ref[:, 0], atol=1e-10, rtol=1e-10)
    np.testing.assert_allclose(S, S_ref[0], atol=1e-10, rtol=1e-10)


def test_gated_chunk_form_strong_gates():
    """Strong per-token decays (down to log_alpha = -10) stay finite through
    the sub-chunk factorisation and still match the recurrence."""
    rng = np.random.default_rng(5)
    T, dk, dv = 128, 16, 8
    q, k, v, _, b = _rand_case(rng, T, 1, dk, dv)
    la = -rng.uniform(0.0, 10.0, size=(T, 1, dk))
    S0 = rng.standard_normal((dk, dv))
    O_ref, S_ref = _fwd(q, k, v, la, b, S0[None])
    O, S = ca.chunk_kda_gated(q[:, 0], k[:, 0], v[:, 0], la[:, 0], b[:, 0], 64, S0, 16)
    assert np.isfinite(O).all() and np.isfinite(S).all()
    np.testing.assert_allclose(O, O_ref[:, 0], atol=1e-9)
    np.testing.assert_allclose(S, S_ref[0], atol=1e-9)


def test_block_inverse_matches_dense():
    rng = np.random.default_rng(3)
    for L in (64, 50, 16, 1):
        N = np.tril(rng.standard_normal((L, L)) * 0.3, -1)
        X = ca.block_unit_lower_inverse(N, 16)
        np.testing.assert_allclose(X @ (np.eye(L) + N), np.eye(L), atol=1e-10)


# ---------------------------------------------------------------------------
# Bounds, decode, multi-sequence packing, golden values
# ---------------------------------------------------------------------------

def test_stability_bound():
    """Unit keys, beta in [0,1], alpha in [0,1]: the transition
    (I - b k k^T) Diag(alpha) is non-expansive, so
    ||S_t||_2 <= ||S_{t-1}||_2 + b ||v_t||."""
    rng = np.random.default_rng(11)
    T, dk, dv = 40, 8, 8
    q, k, v, la, b = _rand_case(rng, T, 1, dk, dv)
    S = rng.standard_normal((dk, dv))
    for t in range(T):
        _, S_next = _fwd(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], b[t:t + 1], S[None])
        S_next = S_next[0]
        assert np.linalg.norm(S_next, 2) <= np.linalg.norm(S, 2) + b[t, 0] * np.linalg.norm(v[t, 0]) + 1e-12
        S = S_next


def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(2)
    T, B, H, dk, dv = 6, 3, 2, 5, 4
    q, k, v, la, b = (np.stack(x) for x in zip(*[_rand_case(rng, T, H, dk, dv) for _ in range(B)]))
    S0 = rng.standard_normal((B, H, dk, dv))
    o_pre, S_pre = oracle.kda_forward(q, k, v, la, b, init_state=S0)
    S = S0
    for t in range(T):
        o_t, S = oracle.kda_decode_step(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], S)
        np.testing.assert_array_equal(o_t, o_pre[:, t])
    np.testing.assert_array_equal(S, S_pre)


def test_packed_sequences_are_independent():
    rng = np.random.default_rng(4)
    lens = [5, 0, 9, 1]
    H, dk, dv = 2, 4, 3
    cases = [_rand_case(rng, L, H, dk, dv) for L in lens]
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    cat = [np.concatenate([c[i] for c in cases]) for i in range(5)]
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, fin = oracle.kda_forward(*cat, init_state=S0, cu_seqlens=cu)
    for i, (c, L) in enumerate(zip(cases, lens)):
        oi, Si = _fwd(*c, S0[i])
        np.testing.assert_array_equal(o[cu[i]:cu[i + 1]], oi)
        np.testing.assert_array_equal(fin[i], Si)
    np.testing.assert_array_equal(fin[1], S0[1])   # empty sequence: state passes through


def test_thread_count_does_not_change_result():
    rng = np.random.default_rng(9)
    q, k, v, la, b = _rand_case(rng, 30, 6, 8, 8)
    o1, s1 = oracle.kda_forward(q, k, v, la, b, n_threads=1)
    o8, s8 = oracle.kda_forward(q, k, v, la, b, n_threads=8)
    np.testing.assert_array_equal(o1, o8)
    np.testing.assert_array_equal(s1, s8)


def test_golden_unit_key_retrieval():
    """Hand-worked values from the retrieval example of "DeltaNet, or Fast
    Weight Programmers": one association written from an empty state is read
    back at the same key scaled by the key's squared norm; a unit key returns
    the value itself; a second write to the same key overwrites it."""
    with open(os.path.join(GOLDEN, "unit_key_retrieval.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        q = np.array(case["q"], dtype=np.float64)[:, None, :]
        k = np.array(case["k"], dtype=np.float64)[:, None, :]
        v = np.array(case["v"], dtype=np.float64)[:, None, :]
        b = np.array(case["beta"], dtype=np.float64)[:, None]
        la = np.zeros_like(k)
        o, S = _fwd(q, k, v, la, b)
        np.testing.assert_allclose(o[:, 0], np.array(case["o"]), atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(S[0], np.array(case["S"]), atol=1e-12, err_msg=case["name"])


def test_golden_channel_gate():
    """Hand-worked values for the channel-wise gate ("Gated Delta Net", "KDA /
    Kimi Linear"): each key row of the state decays by its own alpha before the
    key reads it, alpha = 0 clears only its row, and the read-out comes after
    the write."""
    with open(os.path.join(GOLDEN, "channel_gate.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        q = np.array(case["q"], dtype=np.float64)[:, None, :]
        k = np.array(case["k"], dtype=np.float64)[:, None, :]
        v = np.array(case["v"], dtype=np.float64)[:, None, :]
        b = np.array(case["beta"], dtype=np.float64)[:, None]
        with np.errstate(divide="ignore"):
            la = np.log(np.array(case["alpha"], dtype=np.float64))[:, None, :]   # log 0 = -inf
        S0 = None
        if "S0" in case:
            S0 = np.array(case["S0"], dtype=np.float64)[None, None]
        o, S = oracle.kda_forward(q, k, v, la, b, init_state=S0)
        np.testing.assert_allclose(o[:, 0], np.array(case["o"]), atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(S[0, 0], np.array(case["S"]), atol=1e-12, err_msg=case["name"])


# ---------------------------------------------------------------------------
# The pins are sharp: planted mistakes (in Python copies of the loop) fail them
# ---------------------------------------------------------------------------

def _loop(q, k, v, la, b, S0=None, mistake=None):
    T, H, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((H, dk, dv)) if S0 is None else S0.copy()
    o = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            a = np.exp(la[t, h])
            if mistake == "gate_on_value_columns":
                Sd = S[h] * np.resize(a, dv)[None, :]
            else:
                Sd = a[:, None] * S[h]
            r = (S[h] if mistake == "read_before_decay" else Sd).T @ k[t, h]
            beta = 1.0 if mistake == "drop_beta" else b[t, h]
            d = beta * (v[t, h] - r)
            if mistake == "delta_sign":
                d = -d
            Snew = Sd + np.outer(k[t, h], d)
            o[t, h] = (Sd if mistake == "readout_before_write" else Snew).T @ q[t, h]
            S[h] = Snew
    return o, S


@pytest.mark.parametrize("mistake", ["read_before_decay", "gate_on_value_columns",
                                     "readout_before_write", "drop_beta", "delta_sign"])
def test_pins_catch_planted_mistakes(mistake):
    def fwd(q, k, v, la, b, S0=None):
        o, S = _loop(q, k, v, la, b, S0, mistake)
        return o, S
    failures = 0
    for pin in PINS:
        try:
            pin(fwd, np.random.default_rng(1234))
        except (AssertionError, ValueError, IndexError):
            failures += 1
    assert failures >= 1, "no pin caught the planted mistake %s" % mistake


def test_python_loop_without_mistake_passes_pins():
    for pin in PINS:
        pin(lambda *a: _loop(*a), np.random.default_rng(1234))
