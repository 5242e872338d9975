"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Page titles (cited in short form below):
  "Ten questions"   会加减乘除就够:十个问题,手算读懂 Kimi K3 心脏里的全部数学 (jokeuncle.github.io)
  "22,580"          22,580：从 GPT-2 到 Kimi K3 —— 大模型架构七年进化全解 (yichencityu.github.io)
  "aidehub"         the aidehub.top summary of the same worklog
  "KDA bra-ket blog" the translated blog on the DeltaNet family (mynewscn.com)

Every pin is written as a function of a runner ``run(q, k, v, la, beta, S0, cu,
scale) -> (o, S_final)`` so that the same pins can be shown to catch planted
mistakes in a small pure-Python mirror (``test_pins_catch_planted_mistakes``).
"""
import math

import numpy as np
import pytest

import oracle
from oracle.chunked import chunk_terms, chunked_single
from gated_delta_rule_119_b200.inputs import (bf16_bits_to_f32, f32_to_bf16_bits, make_inputs,
                                             storage_to_f64)
from tests.golden_io import load_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def c_run(q, k, v, la, beta, S0=None, cu=None, scale=1.0):
    return oracle.recurrent_full(q, k, v, la, beta, S0, cu, scale=scale)


def one_head(*xs):
    """[T, d] -> [T, 1, d] (and [T] -> [T, 1])."""
    out = []
    for x in xs:
        x = np.asarray(x, dtype=np.float64)
        out.append(x[:, None, :] if x.ndim == 2 else x[:, None])
    return out


def state1(S):
    return np.asarray(S, dtype=np.float64)[None, None]


# --------------------------------------------------------------------------- pins
def pin_store_retrieve(run):
    """"Ten questions" Q3-Q4: store cat->fish, read it back."""
    g = load_golden("q3q4_store_retrieve.txt")
    q, k, v, la = one_head([g["q"]], [g["k"]], [g["v"]], [[0.0, 0.0]])
    (beta,) = one_head([1.0])
    o, S = run(q, k, v, la, beta, None, None, 1.0)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-15)
    np.testing.assert_allclose(o[0, 0], g["o"], atol=1e-15)


def pin_crosstalk(run):
    """"Ten questions" Q5: purely additive memory mixes fish with 0.6 bone.

    The oracle has no purely additive mode; with beta = eps and values scaled
    by 1/eps the delta rule tends to plain accumulation with an O(eps) error."""
    g = load_golden("q5_crosstalk.txt")
    eps = 1e-7
    q, k, v, la = one_head([g["q"], g["q"]], [g["k1"], g["k2"]],
                           [g["v1"] / eps, g["v2"] / eps], np.zeros((2, 2)))
    (beta,) = one_head([eps, eps])
    o, S = run(q, k, v, la, beta, None, None, 1.0)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-6)
    np.testing.assert_allclose(o[1, 0], g["o"], atol=1e-6)
    # brute force causal sum of the same two writes: sum_i (k_i . q) v_i
    brute = sum(np.dot(ki, g["q"]) * vi for ki, vi in ((g["k1"], g["v1"]), (g["k2"], g["v2"])))
    np.testing.assert_allclose(o[1, 0], brute, atol=1e-6)


def pin_crosstalk_delta(run):
    """The same two writes with the delta rule at beta = 1 (derived by hand):
    dog's read of the first state is [0, 0.6], so u = [1, -0.6] and
    S = [[0.6, 0.64], [0.8, -0.48]]; reading dog then returns bone exactly."""
    g = load_golden("q5_crosstalk.txt")
    q, k, v, la = one_head([g["k1"], g["k2"]], [g["k1"], g["k2"]], [g["v1"], g["v2"]],
                           np.zeros((2, 2)))
    (beta,) = one_head([1.0, 1.0])
    o, S = run(q, k, v, la, beta, None, None, 1.0)
    np.testing.assert_allclose(S[0, 0], [[0.6, 0.64], [0.8, -0.48]], atol=1e-15)
    np.testing.assert_allclose(o[1, 0], g["v2"], atol=1e-15)


def pin_delta_correction(run):
    """"Ten questions" Q6: rewrite cat -> yarn ball, beta = 1 and beta = 0.5."""
    g = load_golden("q6_delta_correction.txt")
    q, k, v, la = one_head([g["q"]], [g["k"]], [g["v"]], [[0.0, 0.0]])
    for b, key in ((1.0, "o_beta1"), (0.5, "o_beta05")):
        (beta,) = one_head([b])
        o, S = run(q, k, v, la, beta, state1(g["S0"]), None, 1.0)
        np.testing.assert_allclose(o[0, 0], g[key], atol=1e-15)
        if b == 1.0:
            np.testing.assert_allclose(S[0, 0], g["S_beta1"], atol=1e-15)


def pin_gradient_table(run):
    """"Ten questions" Q7: the printed descent 0 -> 1.5 -> 2.25 -> 2.625 is the
    one-cell delta rule with k = 1, v = 3, beta = 0.5."""
    g = load_golden("q7_gradient_steps.txt")
    n = len(g["steps"])
    q, k, v, la = one_head(np.ones((n, 1)), np.full((n, 1), g["k"]), np.full((n, 1), g["v"]),
                           np.zeros((n, 1)))
    (beta,) = one_head(np.full(n, g["beta"]))
    o, S = run(q, k, v, la, beta, state1(np.reshape(g["s0"], (1, 1))), None, 1.0)
    np.testing.assert_allclose(o[:, 0, 0], g["steps"], atol=1e-15)


def pin_gradient_step(run):
    """"Ten questions" Q7: one step is gradient descent with learning rate beta on
    L(S) = 1/2 |S~^T k - v|^2 (gradient taken by central differences here)."""
    rng = np.random.default_rng(7)
    dk, dv = 3, 2
    S0 = rng.standard_normal((dk, dv))
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(dv)
    la = -rng.random(dk)
    b = 0.37
    q, kk, vv, lla = one_head([np.zeros(dk)], [k], [v], [la])
    (beta,) = one_head([b])
    _, S = run(q, kk, vv, lla, beta, state1(S0), None, 1.0)
    St = np.exp(la)[:, None] * S0
    loss = lambda M: 0.5 * np.sum((M.T @ k - v) ** 2)
    grad = np.zeros_like(St)
    h = 1e-6
    for i in range(dk):
        for j in range(dv):
            E = np.zeros_like(St)
            E[i, j] = h
            grad[i, j] = (loss(St + E) - loss(St - E)) / (2 * h)
    np.testing.assert_allclose(S[0, 0], St - b * grad, atol=1e-8)


def pin_channel_decay(run):
    """"Ten questions" Q8: per-channel (per-row) decay Diag(alpha) S."""
    g = load_golden("q8_channel_decay.txt")
    q, k, v, la = one_head(np.zeros((1, 2)), np.zeros((1, 2)), np.zeros((1, 2)),
                           [np.log(g["alpha"])])
    (beta,) = one_head([0.0])
    _, S = run(q, k, v, la, beta, state1(g["S0"]), None, 1.0)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-15)


def pin_exact_overwrite(run):
    """Unit keys and beta = 1 make the read of the key just written return its
    value exactly ("22,580" §5.1; "Ten questions" Q6), whatever alpha and S."""
    rng = np.random.default_rng(11)
    T, dk, dv = 20, 6, 5
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    la = -rng.random((T, dk)) * 2
    q, kk, vv, lla = one_head(k, k, v, la)
    (beta,) = one_head(np.ones(T))
    o, _ = run(q, kk, vv, lla, beta, state1(rng.standard_normal((dk, dv))), None, 1.0)
    np.testing.assert_allclose(o[:, 0], v, atol=1e-12)


def pin_linear_attention_orthonormal(run):
    """alpha = 1 and orthonormal keys: no read ever sees an earlier key, so the
    state is sum_i beta_i k_i v_i^T and o_t = sum_{i<=t} beta_i (k_i . s q_t) v_i
    (the unnormalised linear attention of the KDA bra-ket blog §1.1)."""
    rng = np.random.default_rng(3)
    dk, dv = 8, 4
    T = dk
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T]
    q = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    b = rng.random(T)
    s = 0.3
    qq, kk, vv, la = one_head(q, k, v, np.zeros((T, dk)))
    (beta,) = one_head(b)
    o, _ = run(qq, kk, vv, la, beta, None, None, s)
    brute = np.array([sum(b[i] * np.dot(k[i], s * q[t]) * v[i] for i in range(t + 1))
                      for t in range(T)])
    np.testing.assert_allclose(o[:, 0], brute, atol=1e-12)


def pin_linear_attention_limit(run):
    """Random keys, alpha = 1, beta -> 0: o / beta tends to the causal sum
    sum_{i<=t} (k_i . s q_t) v_i of plain linear attention."""
    rng = np.random.default_rng(5)
    T, dk, dv = 12, 5, 3
    k = rng.standard_normal((T, dk))
    q = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    eps = 1e-8
    qq, kk, vv, la = one_head(q, k, v, np.zeros((T, dk)))
    (beta,) = one_head(np.full(T, eps))
    o, _ = run(qq, kk, vv, la, beta, None, None, 1.0)
    brute = np.array([sum(np.dot(k[i], q[t]) * v[i] for i in range(t + 1)) for t in range(T)])
    np.testing.assert_allclose(o[:, 0] / eps, brute, rtol=1e-5, atol=1e-5)


def pin_clear(run):
    """alpha = 0 clears the memory ("22,580" §08): S_t = beta_t k_t v_t^T."""
    rng = np.random.default_rng(9)
    T, dk, dv = 6, 4, 3
    q, k, v = (rng.standard_normal((T, d)) for d in (dk, dk, dv))
    b = rng.random(T)
    qq, kk, vv, la = one_head(q, k, v, np.full((T, dk), -np.inf))
    (beta,) = one_head(b)
    o, S = run(qq, kk, vv, la, beta, state1(rng.standard_normal((dk, dv))), None, 0.5)
    np.testing.assert_allclose(S[0, 0], b[-1] * np.outer(k[-1], v[-1]), atol=1e-14)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], (b[t] * np.outer(k[t], v[t])).T @ (0.5 * q[t]),
                                   atol=1e-14)


def pin_cumulative_decay(run):
    """aidehub "Gated DeltaNet": a value written at step x and read at x + t has
    been scaled by the product of the decays of steps x+1 .. x+t (the write's own
    decay is applied before the write)."""
    rng = np.random.default_rng(13)
    T, dk, dv, x = 9, 3, 2, 3
    k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    la = -rng.random((T, dk))
    b = np.zeros(T)
    b[x] = 0.8
    qq, kk, vv, lla = one_head(np.zeros((T, dk)), k, v, la)
    (beta,) = one_head(b)
    _, S = run(qq, kk, vv, lla, beta, None, None, 1.0)
    expect = np.exp(la[x + 1:].sum(axis=0))[:, None] * (0.8 * np.outer(k[x], v[x]))
    np.testing.assert_allclose(S[0, 0], expect, atol=1e-15)


def pin_matrix_form(run):
    """The product form S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T, o = S^T (s q)
    ("Ten questions" intro and 终局), evaluated with dense matrices."""
    rng = np.random.default_rng(17)
    T, dk, dv = 7, 4, 3
    q, k, v = (rng.standard_normal((T, d)) for d in (dk, dk, dv))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    la, b, S0 = -rng.random((T, dk)), rng.random(T), rng.standard_normal((dk, dv))
    qq, kk, vv, lla = one_head(q, k, v, la)
    (beta,) = one_head(b)
    o, S = run(qq, kk, vv, lla, beta, state1(S0), None, 0.5)
    M = S0.copy()
    for t in range(T):
        M = (np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t])) @ M \
            + b[t] * np.outer(k[t], v[t])
        np.testing.assert_allclose(o[t, 0], M.T @ (0.5 * q[t]), atol=1e-13)
    np.testing.assert_allclose(S[0, 0], M, atol=1e-13)


def pin_scale(run):
    """o is linear in the query scale s; the state does not depend on it."""
    rng = np.random.default_rng(19)
    T, dk, dv = 5, 4, 3
    q, k, v = (rng.standard_normal((T, d)) for d in (dk, dk, dv))
    qq, kk, vv, la = one_head(q, k, v, -rng.random((T, dk)))
    (beta,) = one_head(rng.random(T))
    o1, S1 = run(qq, kk, vv, la, beta, None, None, 1.0)
    o2, S2 = run(qq, kk, vv, la, beta, None, None, 0.25)
    np.testing.assert_allclose(o2, 0.25 * o1, atol=1e-14)
    np.testing.assert_allclose(S2, S1, atol=0)


def pin_varlen(run):
    """Packed sequences restart from their own state: packed == one by one."""
    rng = np.random.default_rng(23)
    H, dk, dv = 2, 4, 3
    cu = np.array([0, 5, 6, 13])
    T = cu[-1]
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v, la = rng.standard_normal((T, H, dv)), -rng.random((T, H, dk))
    b = rng.random((T, H))
    S0 = rng.standard_normal((3, H, dk, dv))
    o, S = run(q, k, v, la, b, S0, cu, 0.5)
    for n in range(3):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = run(q[sl], k[sl], v[sl], la[sl], b[sl], S0[n:n + 1], None, 0.5)
        np.testing.assert_allclose(o[sl], on, atol=1e-14)
        np.testing.assert_allclose(S[n], Sn[0], atol=1e-14)


PINS = [pin_store_retrieve, pin_crosstalk, pin_crosstalk_delta, pin_delta_correction,
        pin_gradient_table, pin_gradient_step, pin_channel_decay, pin_exact_overwrite,
        pin_linear_attention_orthonormal, pin_linear_attention_limit, pin_clear,
        pin_cumulative_decay, pin_matrix_form, pin_scale, pin_varlen]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(c_run)


# ------------------------------------------------------- structure of the oracle
def test_default_scale_is_inverse_sqrt_dk():
    rng = np.random.default_rng(29)
    T, H, dk, dv = 4, 1, 16, 2
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v, la, b = rng.standard_normal((T, H, dv)), -rng.random((T, H, dk)), rng.random((T, H))
    o_def, _ = oracle.recurrent_full(q, k, v, la, b)
    o_one, _ = oracle.recurrent_full(q, k, v, la, b, scale=1.0)
    np.testing.assert_allclose(o_def, o_one / math.sqrt(dk), atol=1e-14)


def test_affine_in_initial_state():
    rng = np.random.default_rng(31)
    T, H, dk, dv = 9, 2, 4, 3
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v, la, b = rng.standard_normal((T, H, dv)), -rng.random((T, H, dk)), rng.random((T, H))
    S1, S2 = rng.standard_normal((1, H, dk, dv)), rng.standard_normal((1, H, dk, dv))
    run = lambda S0: oracle.recurrent_full(q, k, v, la, b, S0)
    o0, F0 = run(np.zeros_like(S1))
    o1, F1 = run(S1)
    o2, F2 = run(S2)
    o3, F3 = run(2.0 * S1 - 0.5 * S2)
    np.testing.assert_allclose(o3 - o0, 2.0 * (o1 - o0) - 0.5 * (o2 - o0), atol=1e-12)
    np.testing.assert_allclose(F3 - F0, 2.0 * (F1 - F0) - 0.5 * (F2 - F0), atol=1e-12)


def test_split_run_resumes():
    """Running T1 tokens, then T2 tokens from the returned state == T1 + T2."""
    inp = make_inputs(1, 40, 2, 8, 4, "f32", 41, state=True)
    a = [storage_to_f64(x, "f32") for x in (inp.q, inp.k, inp.v)]
    o, S = oracle.recurrent_full(*a, inp.log_alpha, inp.beta, inp.S0)
    cut = 17
    pre = [x[:cut] for x in (*a, inp.log_alpha, inp.beta)]
    post = [x[cut:] for x in (*a, inp.log_alpha, inp.beta)]
    o1, S1 = oracle.recurrent_full(*pre, inp.S0)
    o2, S2 = oracle.recurrent_full(*post, S1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, atol=1e-13)
    np.testing.assert_allclose(S2, S, atol=1e-13)


def test_single_token_steps_equal_prefill():
    """T one-token calls carrying the state == one T-token call (decode == prefill)."""
    inp = make_inputs(1, 12, 3, 8, 8, "bf16", 43, state=True)
    o, S = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)
    St = inp.S0.astype(np.float64)
    for t in range(12):
        ot, St = oracle.recurrent_full(inp.q[t:t + 1], inp.k[t:t + 1], inp.v[t:t + 1],
                                       inp.log_alpha[t:t + 1], inp.beta[t:t + 1], St)
        np.testing.assert_allclose(ot[0], o[t], atol=1e-13)
    np.testing.assert_allclose(St, S, atol=1e-13)


def test_bf16_inputs_are_widened_exactly():
    """uint16 (bf16 bits) inputs give the same result as their exact fp64 values."""
    inp = make_inputs(2, 10, 2, 8, 4, "bf16", 47)
    o1, S1 = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)
    w = [storage_to_f64(x, "bf16") for x in (inp.q, inp.k, inp.v)]
    o2, S2 = oracle.recurrent_full(*w, inp.log_alpha.astype(np.float64),
                                   inp.beta.astype(np.float64))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_bf16_rounding_is_nearest_even():
    # bf16 keeps 7 fraction bits: the spacing above 1.0 is 2**-7.
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20],
                 dtype=np.float32)
    back = bf16_bits_to_f32(f32_to_bf16_bits(x))
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7],
                                                 np.float32))


def test_oracle_task_subset_matches_full():
    inp = make_inputs(3, 20, 4, 8, 8, "bf16", 53, state=True)
    o, S = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                                 inp.offsets())
    tasks = [(2, 1), (0, 3)]
    outs, sts = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                                 inp.offsets(), tasks=tasks, nthreads=2)
    cu = inp.offsets()
    for (n, h), on, sn in zip(tasks, outs, sts):
        np.testing.assert_array_equal(on, o[cu[n]:cu[n + 1], h])
        np.testing.assert_array_equal(sn, S[n, h])


def test_oracle_rejects_bad_arguments():
    z = np.zeros((2, 1, 2))
    with pytest.raises(ValueError):
        oracle.recurrent(z, z, z, z, np.zeros((2, 1)), None, [0, 3])   # offset past the end
    with pytest.raises(ValueError):
        oracle.recurrent(z, z, z, z, np.zeros((2, 1)), None, None, tasks=[(0, 5)])


# ---------------------------------------------- chunked form == recurrent form
@pytest.mark.parametrize("C", [1, 2, 3, 16, 64, 130])
def test_chunked_equals_recurrent(C):
    """"22,580" §6.2-6.3: chunking reorders the sum exactly, for any chunk size
    (partial last chunks, nonzero initial state, per-channel decay)."""
    inp = make_inputs(1, 130, 1, 16, 8, "f32", 59, state=True)
    q, k, v = (storage_to_f64(x, "f32")[:, 0] for x in (inp.q, inp.k, inp.v))
    la, b, S0 = inp.log_alpha[:, 0].astype(np.float64), inp.beta[:, 0].astype(np.float64), \
        inp.S0[0, 0].astype(np.float64)
    o_ref, S_ref = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)
    o, S = chunked_single(q, k, v, la, b, S0, C)
    np.testing.assert_allclose(o, o_ref[:, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=0, atol=1e-12)


def test_chunked_strong_decay():
    """Decays as strong as the extremes workload (log alpha down to -6 per step)
    are exact in fp64 in the chunked form too."""
    inp = make_inputs(1, 100, 2, 8, 4, "f32", 61, gates="extremes", state=True)
    o_ref, S_ref = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)
    for h in range(2):
        q, k, v = (storage_to_f64(x, "f32")[:, h] for x in (inp.q, inp.k, inp.v))
        o, S = chunked_single(q, k, v, inp.log_alpha[:, h], inp.beta[:, h], inp.S0[0, h], 64)
        scale = np.abs(o_ref[:, h]).max()
        np.testing.assert_allclose(o, o_ref[:, h], rtol=0, atol=1e-12 * scale)
        np.testing.assert_allclose(S, S_ref[0, h], rtol=0, atol=1e-12)


def test_ut_transform_is_the_inverse():
    """T (I + A) = I with A strictly lower triangular ("22,580" §6.3)."""
    rng = np.random.default_rng(67)
    n, dk, dv = 64, 16, 8
    k = rng.standard_normal((n, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    m = chunk_terms(k, rng.standard_normal((n, dv)), -rng.random((n, dk)), rng.random(n),
                    rng.standard_normal((n, dk)), 0.25)
    np.testing.assert_allclose(m["T"] @ (np.eye(n) + m["A"]), np.eye(n), atol=1e-12)
    assert np.all(np.triu(m["A"]) == 0)
    np.testing.assert_allclose(np.diag(m["T"]), 1.0)


# -------------------------------------------- the pins catch planted mistakes
def mirror(q, k, v, la, beta, S0=None, cu=None, scale=1.0, mutation=None):
    """A small pure-Python copy of the recurrence with one planted mistake."""
    q, k, v, la, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, la, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = [0, T] if cu is None else list(cu)
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    Sf = np.zeros((N, H, dk, dv))
    for h in range(H):
        S = np.zeros((dk, dv))
        for n in range(N):
            if mutation != "state_not_reset" or n == 0:
                S = np.zeros((dk, dv)) if S0 is None or mutation == "ignore_S0" else \
                    np.array(S0[n, h], dtype=np.float64)
            for t in range(cu[n], cu[n + 1]):
                a = np.exp(la[t, h] if mutation != "decay_of_previous_token"
                           else (la[t - 1, h] if t > cu[n] else np.zeros(dk)))
                kt, vt, b = k[t, h], v[t, h], beta[t, h]
                qt = (1.0 if mutation == "ignore_scale" else scale) * q[t, h]
                if mutation == "no_decay":
                    a = np.ones(dk)
                if mutation == "decay_columns":
                    S = S * a[None, :dv]
                elif mutation != "decay_after_write":
                    S = a[:, None] * S
                r = S @ kt[:dv] if mutation == "lookup_untransposed" else S.T @ kt
                if mutation == "wrong_sign":
                    u = b * (r - vt)
                elif mutation == "no_beta":
                    u = vt - r
                elif mutation == "beta_on_lookup_only":
                    u = vt - b * r
                else:
                    u = b * (vt - r)
                S_new = S + (np.outer(u, kt) if mutation == "write_transposed"
                             else np.outer(kt, u))
                if mutation == "decay_after_write":
                    S_new = a[:, None] * S_new
                read = S if mutation == "read_before_write" else S_new
                o[t, h] = read @ qt[:dv] if mutation == "readout_untransposed" else read.T @ qt
                S = S_new
            Sf[n, h] = S
    return o, Sf


MUTATIONS = ["no_decay", "decay_columns", "decay_after_write", "decay_of_previous_token",
             "lookup_untransposed", "readout_untransposed", "wrong_sign", "no_beta",
             "beta_on_lookup_only", "write_transposed", "read_before_write", "ignore_scale",
             "ignore_S0", "state_not_reset"]


def test_pins_pass_on_the_unmutated_mirror():
    for pin in PINS:
        pin(mirror)


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_pins_catch_planted_mistakes(mutation):
    """Each plausible mistake (dropped term, wrong sign, wrong index, transposed
    operand, skipped reset) fails at least one pin."""
    run = lambda *a: mirror(*a, mutation=mutation)
    failed = []
    for pin in PINS:
        try:
            pin(run)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {mutation!r}"
