"""Pins of the Q8_0 part of the oracle (GGUF Q8_0: 34-byte blocks, f16 d then
32 signed 8-bit codes, weight = q * d), each against something other than
the oracle's own formula: closed forms, an independent numpy dequantisation,
exact rational arithmetic, an independent inverse of the packed layout."""
from fractions import Fraction

import numpy as np

import oracle
import synth
from tests.q4_helpers import f16_bits, f16_values

RNG = np.random.default_rng(8080)


def encode_q8_0(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """GGUF Q8_0 bytes from codes q[N][K] (int) and scale bits d[N][K/32]."""
    N, K = q.shape
    out = np.empty((N, K // 32, 34), dtype=np.uint8)
    out[:, :, 0] = d_bits & 0xFF
    out[:, :, 1] = d_bits >> 8
    out[:, :, 2:] = q.reshape(N, K // 32, 32).astype(np.int8).view(np.uint8)
    return out.reshape(N, -1)


def dequant_numpy(g: np.ndarray, N: int, K: int) -> np.ndarray:
    b = g.reshape(N, K // 32, 34)
    d = b[:, :, :2].copy().view("<f2")[:, :, 0].astype(np.float64)
    q = b[:, :, 2:].copy().view(np.int8).astype(np.float64)
    return (q * d[:, :, None]).reshape(N, K)


def test_zero_codes_give_zero():
    N, K = 8, 96
    g = encode_q8_0(np.zeros((N, K), int), RNG.integers(0x2000, 0x3000, (N, K // 32)).astype(np.uint16))
    x = synth.activations(3, 2, K)
    assert np.all(oracle.q8_gemv(g, K, x) == 0.0)


def test_unit_vectors_pin_code_order_sign_and_scale():
    """x = e_k: y_n = q[n][k] * d exactly; codes include -128, -1, 0, 127."""
    N, K = 5, 64
    q = RNG.integers(-128, 128, (N, K))
    q[0, :4] = [-128, -1, 0, 127]
    d = f16_bits(np.full((N, K // 32), 0.125))
    d[:, 1] = f16_bits(np.full(N, -3.0))
    g = encode_q8_0(q, d)
    for k in (0, 1, 2, 3, 17, 31, 32, 45, 63):
        x = np.zeros(K)
        x[k] = 1.0
        y = oracle.q8_gemv(g, K, f16_bits(x)[None, :])[0]
        scale = 0.125 if k < 32 else -3.0
        assert np.array_equal(y, q[:, k] * scale), k


def test_scale_linearity_powers_of_two():
    N, K = 6, 128
    q = RNG.integers(-128, 128, (N, K))
    d1 = f16_bits(RNG.uniform(0.01, 0.05, (N, K // 32)))
    g1 = encode_q8_0(q, d1)
    g2 = encode_q8_0(q, f16_bits(f16_values(d1) * 4.0))
    x = synth.activations(5, 1, K)
    assert np.array_equal(oracle.q8_gemv(g2, K, x), 4.0 * oracle.q8_gemv(g1, K, x))


def test_exact_rationals_brute_force():
    N, K = 3, 64
    q = RNG.integers(-128, 128, (N, K))
    d = f16_bits(RNG.uniform(-0.05, 0.05, (N, K // 32)))
    g = encode_q8_0(q, d)
    x = synth.activations(9, 1, K)
    y = oracle.q8_gemv(g, K, x)[0]
    dv, xv = f16_values(d), f16_values(x[0])
    for n in range(N):
        exact = sum(Fraction(int(q[n, k])) * Fraction(float(dv[n, k // 32])) * Fraction(float(xv[k]))
                    for k in range(K))
        assert abs(Fraction(y[n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)


def test_dense_equivalence_synthetic_matrix():
    N, K = 40, 256
    g = synth.q8_0_matrix(11, synth.weight_id(3), N, K)
    x = synth.activations(11, 3, K)
    want = f16_values(x) @ dequant_numpy(g, N, K).T
    got = oracle.q8_gemv(g, K, x, threads=4)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def unrepack_q8(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Inverse of the packed Q8_0 layout by array reshapes (independent of the
    oracle's loops): segment = [g][c][i][half][e] codes, then [g][i] scales."""
    KB, T = K // 32, (N + 31) // 32
    seg = packed.reshape(T, KB, 1088)
    codes = seg[:, :, :1024].reshape(T, KB, 8, 4, 4, 2, 4)          # t b g c i half e
    qs = codes.transpose(0, 4, 2, 1, 5, 3, 6).reshape(T, 4, 8, KB, 32)  # t i g b (half c e)
    qs = qs.reshape(T * 32, KB, 32)                                   # row = 32t + 8i + g
    sc = seg[:, :, 1024:].reshape(T, KB, 8, 4, 2).transpose(0, 3, 2, 1, 4).reshape(T * 32, KB, 2)
    return np.concatenate([sc, qs], axis=2).reshape(T * 32, KB * 34)[:N]


def test_repack_q8_round_trip_and_padding():
    N, K = 40, 96
    g = synth.q8_0_matrix(2, synth.weight_id(7), N, K)
    p = oracle.repack_q8(g, N, K)
    assert p.size == oracle.packed_bytes_q8(N, K) == 64 * 3 * 34
    assert np.array_equal(unrepack_q8(p, N, K), g)
    pad = unrepack_q8(p, 64, K)[N:]
    assert np.all(pad == 0)                       # codes 0 and d = +0: zero weights
