"""Pins for the oracle's gate forms and input prologue (kda_forward_ex).

Each check ties the oracle to something other than itself:
  * the plain delta rule (no gate; "DeltaNet, or Fast Weight Programmers"
    section of "22580: from GPT-2 to Kimi K3, explained") against the
    independent ungated chunk algebra (chunk-wise parallel form, section
    "DeltaNet, or Parallelizing Linear Transformers with Delta Rule");
  * the scalar gate of "Gated Delta Net" (one decay multiplying the whole
    previous state) against the ungated recurrence through an exact
    rescaling identity: with A_t the product of the decays up to t, the
    gated state is A_t times the ungated state driven by v_t / A_t;
  * the prologue's elementwise functions against closed forms and
    identities (SiLU, sigmoid, log-sigmoid, unit L2 norm), and the raw-input
    path against the same recurrence run on host-normalised inputs.
"""
import numpy as np
import pytest

import oracle
from tests import chunk_algebra as ca


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_no_gate_equals_the_ungated_chunk_algebra():
    rng = np.random.default_rng(71)
    T, H, dk, dv = 37, 2, 8, 5
    q, k = _unit(rng.standard_normal((T, H, dk))), _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    b = rng.uniform(0, 1, (T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = oracle.kda_forward_ex(q, k, v, None, b, init_state=S0, gate="none")
    for h in range(H):
        o_ref, S_ref = ca.chunk_delta_ungated(q[:, h], k[:, h], v[:, h], b[:, h], C=8,
                                              S0=S0[0, h])
        np.testing.assert_allclose(o[:, h], o_ref, rtol=0, atol=1e-11)
        np.testing.assert_allclose(S[0, h], S_ref, rtol=0, atol=1e-11)


def test_scalar_gate_rescaling_identity():
    """S_t = A_t S~_t and o_t = A_t o~_t, where S~ runs the ungated recurrence
    on v_t / A_t from S0 and A_t = prod_{s<=t} alpha_s (scalar per head)."""
    rng = np.random.default_rng(72)
    T, H, dk, dv = 25, 3, 6, 4
    q, k = _unit(rng.standard_normal((T, H, dk))), _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    b = rng.uniform(0, 1, (T, H))
    la = -rng.uniform(0.0, 0.3, (T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = oracle.kda_forward_ex(q, k, v, la, b, init_state=S0, gate="scalar")
    A = np.exp(np.cumsum(la, axis=0))                       # [T, H]
    o_u, S_u = oracle.kda_forward_ex(q, k, v / A[:, :, None], None, b, init_state=S0,
                                     gate="none")
    np.testing.assert_allclose(o, A[:, :, None] * o_u, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S[0], A[-1][:, None, None] * S_u[0], rtol=1e-10, atol=1e-12)


def test_scalar_gate_decays_every_key_row_alike():
    """A scalar gate of exactly -inf clears the whole state; of log(1/2)
    halves it before the read (beta = 0: pure decay)."""
    rng = np.random.default_rng(73)
    H, dk, dv = 2, 4, 3
    S0 = rng.standard_normal((1, H, dk, dv))
    q, k = _unit(rng.standard_normal((1, H, dk))), _unit(rng.standard_normal((1, H, dk)))
    v = rng.standard_normal((1, H, dv))
    _, S = oracle.kda_forward_ex(q, k, v, np.full((1, H), np.log(0.5)), np.zeros((1, H)),
                                 init_state=S0, gate="scalar")
    np.testing.assert_allclose(S, 0.5 * S0, rtol=1e-15)
    b = rng.uniform(0.1, 1, (1, H))
    _, S = oracle.kda_forward_ex(q, k, v, np.full((1, H), -np.inf), b, init_state=S0,
                                 gate="scalar")
    np.testing.assert_allclose(S[0], b[0][:, None, None] * k[0][:, :, None] * v[0][:, None, :],
                               rtol=1e-14)


def test_gate_shapes_are_checked():
    x = np.zeros((3, 2, 4))
    with pytest.raises(ValueError):
        oracle.expand_gate(np.zeros((3, 2)), "channel", (3, 2), 4)
    with pytest.raises(ValueError):
        oracle.expand_gate(x, "scalar", (3, 2), 4)
    with pytest.raises(ValueError):
        oracle.expand_gate(x, "diagonal", (3, 2), 4)


def test_elementwise_closed_forms():
    x = np.array([-800.0, -30.0, -2.5, -1e-3, 0.0, 1e-3, 2.5, 30.0, 800.0])
    s = oracle.sigmoid(x)
    assert s[4] == 0.5
    np.testing.assert_allclose(s + oracle.sigmoid(-x), 1.0, rtol=0, atol=1e-15)
    assert s[0] == 0.0 and s[-1] == 1.0
    ls = oracle.log_sigmoid(x)
    np.testing.assert_allclose(ls[4], -np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(ls - oracle.log_sigmoid(-x), x, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(ls[0], -800.0, rtol=1e-15)          # log sigmoid(x) -> x
    np.testing.assert_allclose(ls[-2], -np.exp(-30.0), rtol=1e-10)  # -> -e^-x
    assert np.all(ls <= 0)
    si = oracle.silu(x)
    assert si[4] == 0.0
    np.testing.assert_allclose(si - oracle.silu(-x), x, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(si[-1], 800.0, rtol=1e-15)
    assert si[0] == 0.0 or abs(si[0]) < 1e-300


def test_qk_prologue_has_unit_norm_and_the_normalise_guard():
    rng = np.random.default_rng(74)
    x = rng.standard_normal((50, 3, 16)) * rng.uniform(0.01, 100, (50, 3, 1))
    y = oracle.prologue_qk(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    # normalisation is invariant to a positive scale of the SiLU output
    z = oracle.silu(x)
    np.testing.assert_allclose(oracle.l2_normalize(7.5 * z), oracle.l2_normalize(z), rtol=1e-14)
    # the zero vector stays zero (divided by eps, not by zero)
    assert np.all(oracle.prologue_qk(np.zeros((2, 8))) == 0.0)


@pytest.mark.parametrize("gate", oracle.GATES)
def test_raw_inputs_equal_host_prologue(gate):
    rng = np.random.default_rng(75)
    T, H, dk, dv = 20, 2, 8, 6
    qr, kr = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    bl = rng.standard_normal((T, H))
    gl = rng.standard_normal((T, H, dk) if gate == "channel" else (T, H)) + 3.0
    o, S = oracle.kda_forward_ex(qr, kr, v, gl, bl, gate=gate, raw_qk=True, raw_beta=True,
                                 raw_gate=True)
    q = np.stack([[oracle.l2_normalize(oracle.silu(qr[t, h])) for h in range(H)]
                  for t in range(T)])
    k = np.stack([[oracle.l2_normalize(oracle.silu(kr[t, h])) for h in range(H)]
                  for t in range(T)])
    b = 1.0 / (1.0 + np.exp(-bl))
    la = np.log(1.0 / (1.0 + np.exp(-gl)))
    o2, S2 = oracle.kda_forward_ex(q, k, v, la, b, gate=gate)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-13)
