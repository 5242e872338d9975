"""Pins of the oracle's gate front-ends (oracle/gates.py) against what the pages and the
mathematics fix, with no GPU:

* "Ten questions" Q9's printed values of exp, sigmoid and softplus (tests/golden/q9_squashing.txt);
* the property Q9 states for the gate line g = -exp(A_log) softplus(f + dt_bias): alpha = e^g
  lies in (0, 1) for any input (in [0, 1] once fp64 underflows), and e^A_log scales g;
* softplus and sigmoid against numpy/scipy library routines on a wide range;
* unit-length keys and queries ("22,580" §5.2), scale-invariant, zero vectors kept finite;
* the scalar gate (Gated DeltaNet, "22,580" §08) through a closed form: with one alpha per
  token, S_t / Gamma_t (Gamma_t the running product of alpha) follows the plain delta rule on
  the values v_t / Gamma_t, so the recurrence fed the broadcast gate must equal Gamma_t times
  the no-decay recurrence on rescaled values;
* the fused path equal to the plain recurrence fed the same alpha, and unchanged when the keys
  are scaled before normalisation.
A planted-mistake check confirms each pin catches a plausible slip in the front-end."""
import math

import numpy as np
import pytest

import oracle
from oracle import gates
from tests.golden_io import load_golden


def test_q9_printed_values():
    g = load_golden("q9_squashing.txt")
    fns = {"exp": np.exp, "sigmoid": gates.sigmoid, "softplus": gates.softplus}
    for name, fn in fns.items():
        xs, ys, dec = (np.atleast_1d(g[f"{name}_{s}"]) for s in ("x", "y", "dec"))
        for x, y, d in zip(xs, ys, dec):
            assert round(float(fn(x)), int(d)) == pytest.approx(y, abs=1e-12), (name, x)


def test_softplus_and_sigmoid_match_library_routines():
    from scipy.special import expit
    x = np.linspace(-700.0, 700.0, 20001)
    np.testing.assert_allclose(gates.softplus(x), np.logaddexp(0.0, x), rtol=1e-15, atol=0)
    np.testing.assert_allclose(gates.sigmoid(x), expit(x), rtol=1e-15, atol=1e-300)
    assert np.all(gates.softplus(x) > 0)
    assert np.all(gates.softplus(x) >= np.maximum(x, 0))
    assert np.all(gates.softplus(x) <= np.maximum(x, 0) + math.log(2) + 1e-15)


def test_fused_gate_keeps_alpha_in_the_unit_interval():
    rng = np.random.default_rng(0)
    f = rng.uniform(-40, 40, size=(300, 3, 8))
    A = rng.uniform(-4, 3, size=(3, 8))
    b = rng.uniform(-10, 10, size=(3, 8))
    la = gates.fused_log_alpha(f, A, b)
    alpha = np.exp(la)
    moderate = np.abs(f + b[None]) < 30
    assert np.all((alpha[moderate] > 0) & (alpha[moderate] < 1))
    assert np.all((alpha >= 0) & (alpha <= 1)) and np.all(np.isfinite(la))
    huge = gates.fused_log_alpha(np.array([[[1e4, -1e4]]]), np.array([[5.0, 5.0]]), np.zeros((1, 2)))
    assert np.all(np.exp(huge) >= 0) and np.all(np.exp(huge) <= 1) and np.all(np.isfinite(huge))


def test_fused_gate_structure():
    """exp(A_log) multiplies g (A_log = ln 2 doubles it); dt_bias shifts the pre-activation;
    A_log = dt_bias = 0 is the default gate recipe -softplus(f) of the generator."""
    rng = np.random.default_rng(1)
    f = rng.standard_normal((50, 2, 4))
    base = gates.fused_log_alpha(f, np.zeros((2, 4)), np.zeros((2, 4)))
    np.testing.assert_allclose(base, -np.logaddexp(0.0, f), rtol=1e-15)
    np.testing.assert_allclose(gates.fused_log_alpha(f, np.full((2, 4), math.log(2.0)), np.zeros((2, 4))),
                               2.0 * base, rtol=1e-15)
    d = rng.standard_normal((2, 4))
    np.testing.assert_allclose(gates.fused_log_alpha(f, np.zeros((2, 4)), d),
                               -np.logaddexp(0.0, f + d[None]), rtol=1e-15)


def test_fused_gate_reads_bf16_bits_exactly():
    from gated_delta_rule_119_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits
    rng = np.random.default_rng(2)
    f32 = rng.standard_normal((20, 2, 8)).astype(np.float32)
    bits = f32_to_bf16_bits(f32)
    np.testing.assert_array_equal(gates.widen(bits), bf16_bits_to_f32(bits).astype(np.float64))
    np.testing.assert_array_equal(gates.fused_log_alpha(bits, np.zeros((2, 8)), np.zeros((2, 8))),
                                  gates.fused_log_alpha(bf16_bits_to_f32(bits), np.zeros((2, 8)),
                                                        np.zeros((2, 8))))


def test_l2_normalize():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((30, 2, 16))
    n = gates.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(gates.l2_normalize(7.5 * x), n, rtol=1e-14)
    z = gates.l2_normalize(np.zeros((1, 1, 4)))
    assert np.all(z == 0)


def _scalar_case(seed, T=40, dk=8, dv=6):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, dv))
    la = -rng.uniform(0.0, 0.3, size=(T, 1))
    beta = rng.uniform(0.1, 0.9, size=(T, 1))
    S0 = rng.standard_normal((1, 1, dk, dv))
    return q, k, v, la, beta, S0


def scalar_pin(q, k, v, la, beta, S0, broadcast=gates.broadcast_scalar):
    """Checks recurrent(broadcast scalar gate) == Gamma_t * recurrent(no decay, v / Gamma)."""
    dk = q.shape[-1]
    o, S = oracle.recurrent_full(q, k, v, broadcast(la, dk), beta, S0)
    Gamma = np.exp(np.cumsum(la[:, 0]))                 # running product of alpha
    o1, S1 = oracle.recurrent_full(q, k, v / Gamma[:, None, None], np.zeros(q.shape), beta, S0)
    ok_o = np.allclose(o, Gamma[:, None, None] * o1, rtol=1e-10, atol=1e-12)
    ok_s = np.allclose(S, Gamma[-1] * S1, rtol=1e-10, atol=1e-12)
    return ok_o and ok_s


@pytest.mark.parametrize("seed", [4, 5, 6])
def test_scalar_gate_closed_form(seed):
    assert scalar_pin(*_scalar_case(seed))


def test_no_gate_is_deltanet_exact_overwrite():
    """alpha = 1 (DeltaNet): with unit keys and beta = 1 the state returns v_t for k_t."""
    q, k, v, la, beta, S0 = _scalar_case(7, T=12)
    la0 = gates.broadcast_scalar(np.zeros_like(la), q.shape[-1])
    for t in range(1, 13):
        _, S = oracle.recurrent_full(q[:t], k[:t], v[:t], la0[:t], np.ones((t, 1)), S0)
        np.testing.assert_allclose(S[0, 0].T @ k[t - 1, 0], v[t - 1, 0], atol=1e-12)


def test_fused_path_equals_recurrence_fed_the_same_alpha_and_is_scale_invariant():
    rng = np.random.default_rng(8)
    T, H, dk, dv = 30, 2, 8, 8
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    f = rng.standard_normal((T, H, dk))
    A, b = rng.uniform(-2, 1, (H, dk)), rng.uniform(-1, 1, (H, dk))
    braw = rng.standard_normal((T, H))
    la = gates.fused_log_alpha(f, A, b)
    beta = gates.sigmoid(braw)
    kn, qn = gates.l2_normalize(k), gates.l2_normalize(q)
    o1, S1 = oracle.recurrent_full(qn, kn, v, la, beta)
    o2, S2 = oracle.recurrent_full(gates.l2_normalize(3.0 * q), gates.l2_normalize(0.25 * k), v,
                                   gates.fused_log_alpha(f, A, b), gates.sigmoid(braw))
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-13)


def test_gate_pins_catch_planted_mistakes():
    """Plausible slips in the front-end, each planted in a copy on the CPU, fail a pin."""
    g = load_golden("q9_squashing.txt")

    def printed_ok(softplus, sigmoid):
        ok = all(round(float(softplus(x)), 3) == y for x, y in zip(g["softplus_x"], g["softplus_y"]))
        return ok and all(round(float(sigmoid(x)), int(d)) == y for x, y, d in
                          zip(g["sigmoid_x"], g["sigmoid_y"], g["sigmoid_dec"]))

    assert printed_ok(gates.softplus, gates.sigmoid)
    assert not printed_ok(lambda x: np.exp(x), gates.sigmoid)                  # log dropped
    assert not printed_ok(lambda x: np.log(1 + np.exp(-x)), gates.sigmoid)    # sign flipped inside
    assert not printed_ok(gates.softplus, lambda x: 1 / (1 + np.exp(x)))      # sigmoid sign flipped
    rng = np.random.default_rng(9)
    f, A, b = rng.uniform(-5, 5, (20, 2, 4)), rng.uniform(-2, 2, (2, 4)), rng.uniform(-2, 2, (2, 4))

    def unit_ok(fn):
        a = np.exp(fn(f, A, b))
        return bool(np.all((a > 0) & (a < 1)))

    def scale_ok(fn):
        f0 = rng.standard_normal((10, 2, 4))
        return np.allclose(fn(f0, np.full((2, 4), math.log(2.0)), np.zeros((2, 4))),
                           2 * fn(f0, np.zeros((2, 4)), np.zeros((2, 4))))

    assert unit_ok(gates.fused_log_alpha) and scale_ok(gates.fused_log_alpha)
    assert not unit_ok(lambda f, A, b: np.exp(A)[None] * gates.softplus(f + b[None]))   # minus lost
    assert not scale_ok(lambda f, A, b: -A[None] * gates.softplus(f + b[None]))         # exp(A_log) lost
    # the scalar closed form catches a gate broadcast over the wrong axis or applied twice
    case = _scalar_case(10, dk=8)
    assert not scalar_pin(*case, broadcast=lambda la, dk: np.repeat(la[..., None], dk, -1)[::-1].copy())
    assert not scalar_pin(*case, broadcast=lambda la, dk: 2 * gates.broadcast_scalar(la, dk))
