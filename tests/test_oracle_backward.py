"""Pins for the oracle's reverse mode (oracle.kda_backward): the gradient of
a scalar loss through the token loop, checked against central finite
differences of the forward oracle (fp64, tiny sizes), against closed forms
of special cases, and against planted mistakes.

Loss: L = sum(o * Wo) + sum(S_final * Ws) with fixed random weights, so
dL/do = Wo and dL/dS_final = Ws.
"""
import numpy as np
import pytest

import oracle


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _case(rng, T=6, H=2, dk=5, dv=4, n_seq=1):
    return dict(q=_unit(rng.standard_normal((T, H, dk))), k=_unit(rng.standard_normal((T, H, dk))),
                v=rng.standard_normal((T, H, dv)),
                log_alpha=-rng.uniform(0.0, 1.5, (T, H, dk)),
                beta=rng.uniform(0.1, 1.0, (T, H)),
                init_state=rng.standard_normal((n_seq, H, dk, dv)))


def _loss(inp, Wo, Ws, cu=None):
    o, S = oracle.kda_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              init_state=inp["init_state"], cu_seqlens=cu)
    return float(np.sum(o * Wo) + np.sum(S * Ws))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_matches_finite_differences(seed):
    rng = np.random.default_rng(100 + seed)
    lengths = [4, 0, 3]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    inp = _case(rng, T=sum(lengths), n_seq=len(lengths))
    Wo = rng.standard_normal(inp["v"].shape)
    Ws = rng.standard_normal(inp["init_state"].shape)
    g = oracle.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], Wo,
                            init_state=inp["init_state"], d_final=Ws, cu_seqlens=cu)
    names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta",
             "init_state": "d_init"}
    h = 1e-6
    for name, gname in names.items():
        x = inp[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _loss(inp, Wo, Ws, cu)
            x[idx] = keep - h
            lm = _loss(inp, Wo, Ws, cu)
            x[idx] = keep
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[gname], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_without_writes_or_decay():
    """beta = 0, alpha = 1: nothing is written, o_t = S0^T q_t. So dq_t = S0 do_t,
    dS0 = sum_t q_t do_t^T + dS_final, dv = dk = 0, and dlog_alpha, dbeta follow
    from the gradient G that reaches each S_t (written out below)."""
    rng = np.random.default_rng(7)
    inp = _case(rng, T=5)
    inp["beta"][:] = 0.0
    inp["log_alpha"][:] = 0.0
    Wo = rng.standard_normal(inp["v"].shape)
    Ws = rng.standard_normal(inp["init_state"].shape)
    g = oracle.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], Wo,
                            init_state=inp["init_state"], d_final=Ws)
    S0 = inp["init_state"][0]
    np.testing.assert_allclose(g["dq"], np.einsum("hab,thb->tha", S0, Wo), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(g["d_init"][0], np.einsum("tha,thb->hab", inp["q"], Wo) + Ws[0],
                               rtol=1e-13, atol=1e-13)
    assert np.all(g["dv"] == 0) and np.all(g["dk"] == 0)
    # dlog_alpha_t = sum_j S'[i, j] G'[i, j] with S' = S0 and G' the gradient reaching S_t
    G = Ws[0].copy()
    dla = np.zeros_like(inp["log_alpha"])
    for t in range(4, -1, -1):
        G = G + np.einsum("ha,hb->hab", inp["q"][t], Wo[t])
        dla[t] = np.einsum("hab,hab->ha", S0, G)
    np.testing.assert_allclose(g["dlog_alpha"], dla, rtol=1e-12, atol=1e-12)
    # dbeta_t = (G^T k_t) . (v_t - S0^T k_t)
    G = Ws[0].copy()
    for t in range(4, -1, -1):
        G = G + np.einsum("ha,hb->hab", inp["q"][t], Wo[t])
        dd = np.einsum("hab,ha->hb", G, inp["k"][t])
        r = np.einsum("hab,ha->hb", S0, inp["k"][t])
        np.testing.assert_allclose(g["dbeta"][t], np.sum(dd * (inp["v"][t] - r), -1),
                                   rtol=1e-12, atol=1e-12)


def test_full_clear_cuts_the_gradient_to_the_past():
    """log_alpha = -inf at token t: nothing before t reaches the loss after it."""
    rng = np.random.default_rng(8)
    inp = _case(rng, T=6)
    inp["log_alpha"][3] = -np.inf
    Wo = rng.standard_normal(inp["v"].shape)
    Wo[:3] = 0.0                      # the loss only sees tokens 3..5 and the final state
    Ws = rng.standard_normal(inp["init_state"].shape)
    g = oracle.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], Wo,
                            init_state=inp["init_state"], d_final=Ws)
    for n in ("dq", "dk", "dv", "dbeta"):
        assert np.all(g[n][:3] == 0), n
    assert np.all(g["d_init"] == 0)


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
def test_backward_through_the_prologue_matches_finite_differences(gate):
    """Raw projections (q, k through SiLU and L2 normalisation, beta and gate
    logits through sigmoid and log-sigmoid): oracle.kda_backward_ex against
    central differences of oracle.kda_forward_ex with the same flags."""
    rng = np.random.default_rng(300 + len(gate))
    T, H, dk, dv = 5, 2, 5, 4
    gshape = {"channel": (T, H, dk), "scalar": (T, H), "none": None}[gate]
    inp = dict(q=rng.standard_normal((T, H, dk)), k=rng.standard_normal((T, H, dk)),
               v=rng.standard_normal((T, H, dv)),
               log_alpha=None if gshape is None else rng.standard_normal(gshape) + 1.0,
               beta=rng.standard_normal((T, H)),
               init_state=rng.standard_normal((1, H, dk, dv)))
    Wo = rng.standard_normal((T, H, dv))
    Ws = rng.standard_normal((1, H, dk, dv))
    flags = dict(gate=gate, raw_qk=True, raw_beta=True, raw_gate=True)

    def loss():
        o, S = oracle.kda_forward_ex(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                     inp["beta"], init_state=inp["init_state"], **flags)
        return float(np.sum(o * Wo) + np.sum(S * Ws))

    g = oracle.kda_backward_ex(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], Wo,
                               init_state=inp["init_state"], d_final=Ws, **flags)
    names = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "init_state": "d_init"}
    if gate != "none":
        names["log_alpha"] = "dlog_alpha"
    else:
        assert g["dlog_alpha"] is None
    h = 1e-6
    for name, gname in names.items():
        x = inp[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = loss()
            x[idx] = keep - h
            lm = loss()
            x[idx] = keep
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[gname], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_ex_without_prologue_is_the_plain_reverse_mode():
    """No flags: kda_backward_ex is kda_backward on the expanded gate, with
    the scalar gate's gradient summed over the key channels it was copied to."""
    rng = np.random.default_rng(9)
    T, H, dk, dv = 6, 2, 5, 4
    q, k = _unit(rng.standard_normal((T, H, dk))), _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    la = -rng.uniform(0.0, 1.5, (T, H))
    b = rng.uniform(0.1, 1.0, (T, H))
    s0 = rng.standard_normal((1, H, dk, dv))
    Wo = rng.standard_normal((T, H, dv))
    g = oracle.kda_backward_ex(q, k, v, la, b, Wo, init_state=s0, gate="scalar")
    ref = oracle.kda_backward(q, k, v, np.repeat(la[..., None], dk, -1), b, Wo, init_state=s0)
    for n in ("dq", "dk", "dv", "dbeta", "d_init"):
        np.testing.assert_array_equal(g[n], ref[n])
    np.testing.assert_array_equal(g["dlog_alpha"], ref["dlog_alpha"].sum(-1))


def test_prologue_pin_catches_a_planted_mistake(monkeypatch):
    """The finite-difference pin above is sharp: the normalisation's Jacobian
    without its projection term (a plausible slip) moves dq and dk far
    outside its tolerance."""
    def wrong_vjp(x, g, eps=1e-12):
        x, g = oracle._f64(x), oracle._f64(g)
        s = oracle.sigmoid(x)
        u = x * s
        r = np.sqrt(np.sum(u * u, axis=-1, keepdims=True))
        return g / np.maximum(r, eps) * s * (1.0 + x * (1.0 - s))

    rng = np.random.default_rng(41)
    T, H, dk, dv = 4, 1, 5, 3
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    b = rng.standard_normal((T, H))
    Wo = rng.standard_normal((T, H, dv))

    def loss(qq):
        o, _ = oracle.kda_forward_ex(qq, k, v, None, b, gate="none", raw_qk=True, raw_beta=True)
        return float(np.sum(o * Wo))

    h = 1e-6
    num = np.zeros_like(q)
    for idx in np.ndindex(*q.shape):
        qp, qm = q.copy(), q.copy()
        qp[idx] += h
        qm[idx] -= h
        num[idx] = (loss(qp) - loss(qm)) / (2 * h)
    good = oracle.kda_backward_ex(q, k, v, None, b, Wo, gate="none", raw_qk=True,
                                  raw_beta=True)["dq"]
    np.testing.assert_allclose(good, num, rtol=1e-6, atol=1e-7)
    monkeypatch.setattr(oracle, "_prologue_qk_vjp", wrong_vjp)
    bad = oracle.kda_backward_ex(q, k, v, None, b, Wo, gate="none", raw_qk=True,
                                 raw_beta=True)["dq"]
    assert np.max(np.abs(bad - num)) > 1e-3
