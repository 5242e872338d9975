"""Pins of the oracle's gradients (oracle.backward, reverse mode through the fp64 recurrence)
against what does not depend on its code:

* central finite differences of the forward oracle (oracle.recurrent, itself pinned to the
  pages) on tiny inputs, for every element of every input -- q, k, v, log_alpha, beta, S0 --
  with sequences that cross the backward's 64-token checkpoint segments and a varlen batch;
* exact identities of the recurrence: o is linear in q, and (o, S_final) jointly linear in
  (v, S0), so <dq, q> = sum dO * o and <dv, v> + <dS0, S0> = L for L = sum dO * o +
  sum dS_final * S_final (Euler's theorem for homogeneous functions of degree one);
* alpha = 0 (log_alpha = -inf) gives no gradient to the decay and none past the clearing token.
A mirror with planted slips shows the finite-difference pin catches each of them."""
import numpy as np
import pytest

import oracle


def case(seed, T=9, H=1, dk=3, dv=2, cu=None):
    rng = np.random.default_rng(seed)
    Tt = T if cu is None else cu[-1]
    N = 1 if cu is None else len(cu) - 1
    q = rng.standard_normal((Tt, H, dk))
    k = rng.standard_normal((Tt, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((Tt, H, dv)), log_alpha=-rng.uniform(0.0, 0.8, (Tt, H, dk)),
                beta=rng.uniform(0.1, 0.95, (Tt, H)), S0=rng.standard_normal((N, H, dk, dv))), \
        rng.standard_normal((Tt, H, dv)), rng.standard_normal((N, H, dk, dv))


def loss(x, cu, dO, dSf):
    o, S = oracle.recurrent_full(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu)
    return float((o * dO).sum() + (S * dSf).sum())


def finite_differences(x, cu, dO, dSf, eps=1e-6):
    fd = {}
    for name, a in x.items():
        g = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            y = {kk: vv.copy() for kk, vv in x.items()}
            y[name][i] += eps
            lp = loss(y, cu, dO, dSf)
            y[name][i] -= 2 * eps
            g[i] = (lp - loss(y, cu, dO, dSf)) / (2 * eps)
        fd[name] = g
    return fd


GRAD = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta", "S0": "dS0"}


def assert_matches_fd(grads, fd, tol=2e-8):
    for name, g in fd.items():
        err = np.abs(grads[GRAD[name]] - g).max() / max(np.abs(g).max(), 1e-12)
        assert err < tol, (name, err)


@pytest.mark.parametrize("seed", [0, 1])
def test_gradients_match_finite_differences(seed):
    x, dO, dSf = case(seed)
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], None, dO, dSf)
    assert_matches_fd(g, finite_differences(x, None, dO, dSf))


def test_gradients_across_checkpoint_segments_and_varlen():
    cu = [0, 70, 70, 75]                              # 70 tokens: two 64-token segments; an empty one
    x, dO, dSf = case(2, H=2, dk=2, dv=2, cu=cu)
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu, dO, dSf)
    fd = finite_differences(x, cu, dO, dSf)
    assert_matches_fd(g, fd)
    np.testing.assert_array_equal(g["dS0"][1], dSf[1])   # the empty sequence passes dS_final through


def test_without_final_state_gradient():
    x, dO, _ = case(3)
    zero = np.zeros_like(x["S0"])
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], None, dO, None)
    assert_matches_fd(g, finite_differences(x, None, dO, zero))


def test_homogeneity_identities():
    rng = np.random.default_rng(4)
    T, H, dk, dv = 200, 2, 16, 12
    x, dO, dSf = case(4, T=T, H=H, dk=dk, dv=dv)
    o, S = oracle.recurrent_full(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], None, dO, dSf)
    L = float((o * dO).sum() + (S * dSf).sum())
    np.testing.assert_allclose((g["dq"] * x["q"]).sum(), (o * dO).sum(), rtol=1e-11)
    np.testing.assert_allclose((g["dv"] * x["v"]).sum() + (g["dS0"] * x["S0"]).sum(), L, rtol=1e-11)
    assert rng is not None


def test_clearing_gate_stops_gradients():
    """alpha = 0 at token 4 clears the memory, so with no output gradient before token 4
    nothing before it (inputs of tokens 0-3, S0) and not the clearing gate itself gets any."""
    x, dO, dSf = case(5, T=8)
    x["log_alpha"][4] = -np.inf
    dO[:4] = 0.0
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], None, dO, dSf)
    assert np.all(g["dS0"] == 0) and np.all(g["dlog_alpha"][4] == 0)
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        assert np.all(g[name][:4] == 0), name
    assert np.any(g["dk"][4:] != 0) and np.any(g["dv"][4:] != 0)


def _mirror(x, dO, dSf, slip=None):
    """A pure-Python copy of the reverse step for one pair with an optional planted slip."""
    q, k, v, la, b = (x[n][:, 0] for n in ("q", "k", "v", "log_alpha", "beta"))
    s = q.shape[1] ** -0.5
    T = len(q)
    states = [x["S0"][0, 0].copy()]
    for t in range(T):
        St = np.exp(la[t])[:, None] * states[-1]
        u = b[t] * (v[t] - St.T @ k[t])
        states.append(St + np.outer(k[t], u))
    G = dSf[0, 0].copy()
    out = {n: np.zeros_like(x[n]) for n in x}
    for t in reversed(range(T)):
        G = G + s * np.outer(q[t], dO[t, 0])
        out["q"][t, 0] = s * states[t + 1] @ dO[t, 0]
        St = np.exp(la[t])[:, None] * states[t]
        r = v[t] - St.T @ k[t]
        u = b[t] * r
        du = G.T @ k[t]
        out["v"][t, 0] = (1.0 if slip == "dv_no_beta" else b[t]) * du
        out["beta"][t, 0] = du @ r
        out["k"][t, 0] = G @ u + (1 if slip == "dk_sign" else -1) * b[t] * St @ du
        Gt = G - b[t] * np.outer(k[t], du)
        out["log_alpha"][t, 0] = ((Gt * (states[t] if slip == "dla_prev_state" else St)).sum(1))
        G = (1.0 if slip == "no_decay_back" else np.exp(la[t]))[..., None] * Gt if slip != "no_decay_back" else Gt
    out["S0"][0, 0] = G
    return {GRAD[n]: a for n, a in out.items()}


def test_finite_difference_pin_catches_planted_slips():
    x, dO, dSf = case(6, T=6)
    fd = finite_differences(x, None, dO, dSf)
    assert_matches_fd(_mirror(x, dO, dSf), fd)
    for slip in ("dv_no_beta", "dk_sign", "dla_prev_state", "no_decay_back"):
        with pytest.raises(AssertionError):
            assert_matches_fd(_mirror(x, dO, dSf, slip), fd)
