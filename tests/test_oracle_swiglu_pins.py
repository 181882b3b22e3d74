"""Pins of the SiLU-gated input of the down GEMV in the oracle
(``swiglu``, ``q4_gemv_f64``, ``q4_gemv_swiglu``), each against something
other than the oracle's own formula: the logistic function's symmetry and
Taylor series, its limits, linearity in the up half, agreement with the
already pinned f16-input GEMV, and a dense product from an independent
dequantisation with the gate computed by ``math.exp``."""
import math

import numpy as np

import oracle
import synth
from tests.q4_helpers import f16_bits, f16_values

RNG = np.random.default_rng(4242)


def gate_up(g, p):
    return np.concatenate([f16_bits(np.asarray(g, float)), f16_bits(np.asarray(p, float))])[None, :]


def test_odd_part_of_silu_is_the_identity():
    """silu(x) - silu(-x) = x (sigma(x) + sigma(-x) = 1)."""
    x = f16_values(f16_bits(RNG.normal(0, 4, 4000)))
    g = np.concatenate([x, -x])
    u = oracle.swiglu(gate_up(g, np.ones_like(g)))[0]
    n = x.size
    assert np.allclose(u[:n] - u[n:], x, rtol=4e-16, atol=1e-300)


def test_taylor_series_at_zero_fixes_the_sign_of_the_exponent():
    """sigma(h) = 1/2 + h/4 - h^3/48 + ...: silu(h)/h for small f16 h."""
    h = f16_values(f16_bits(np.array([2.0 ** -6, 2.0 ** -8, -2.0 ** -7, 2.0 ** -10])))
    u = oracle.swiglu(gate_up(h, np.ones_like(h)))[0]
    want = 0.5 + h / 4 - h ** 3 / 48
    assert np.allclose(u / h, want, rtol=0, atol=1e-9)


def test_limits():
    """Large positive gates pass through (silu(g) -> g); large negative ones
    vanish like g e^g; silu(0) = 0."""
    g = np.array([20.0, 40.0, 1000.0, -20.0, -40.0, 0.0, -0.0])
    u = oracle.swiglu(gate_up(g, np.ones_like(g)))[0]
    assert np.allclose(u[:3], g[:3] * (1 - np.exp(-g[:3])), rtol=1e-15)
    ref = g[3:5] * np.exp(g[3:5]) / (1 + np.exp(g[3:5]))
    assert np.allclose(u[3:5], ref, rtol=1e-14)
    assert u[5] == 0.0 and u[6] == 0.0


def test_linear_in_the_up_half_and_gate_is_the_first_half():
    K = 96
    g = RNG.normal(0, 2, K)
    p = RNG.normal(0, 1, K)
    u1 = oracle.swiglu(gate_up(g, p))[0]
    u2 = oracle.swiglu(gate_up(g, 2 * f16_values(f16_bits(p))))[0]
    assert np.array_equal(u2, 2 * u1)
    u0 = oracle.swiglu(gate_up(g, np.zeros(K)))[0]
    assert np.all(u0 == 0.0)
    # the halves are not interchangeable: silu(g) * p != silu(p) * g in general
    assert not np.allclose(oracle.swiglu(gate_up(p, g))[0], u1)


def test_f64_gemv_matches_the_f16_gemv_on_f16_inputs():
    N, K = 40, 256
    rows = synth.q4_0_matrix(3, synth.weight_id(5), N, K)
    x = synth.activations(3, 2, K)
    assert np.array_equal(oracle.q4_gemv_f64(rows, K, f16_values(x)), oracle.q4_gemv(rows, K, x))
    assert np.array_equal(oracle.q4_gemv_f64(rows, K, f16_values(x), threads=4),
                          oracle.q4_gemv(rows, K, x))


def dequant_numpy(g: np.ndarray, N: int, K: int) -> np.ndarray:
    b = g.reshape(N, K // 32, 18)
    d = b[:, :, :2].copy().view("<f2")[:, :, 0].astype(np.float64)
    qs = b[:, :, 2:]
    q = np.concatenate([qs & 0xF, qs >> 4], axis=2).astype(np.float64) - 8
    return (q * d[:, :, None]).reshape(N, K)


def test_gated_gemv_dense_brute_force():
    N, K = 24, 64
    rows = synth.q4_0_matrix(9, synth.weight_id(6), N, K)
    gu = synth.activations(9, 1, 2 * K)
    v = f16_values(gu[0])
    u = np.array([v[k] / (1.0 + math.exp(-v[k])) * v[K + k] for k in range(K)])
    want = dequant_numpy(rows, N, K) @ u
    got = oracle.q4_gemv_swiglu(rows, K, gu)[0]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
