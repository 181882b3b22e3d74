"""Pins for the fp64 oracle and the input generator (no GPU).

Each check ties the oracle to something other than itself: published test
vectors, IEEE-754 tables and numpy's own float16 conversion, closed forms of
the Q4_0 definition (all codes 8, unit vectors, scale linearity), exact
rational brute force from codes chosen by the test, and a closed-form
signed-permutation stack.
"""
from fractions import Fraction
import math

import numpy as np
import pytest

import oracle
import synth
from tests.q4_helpers import encode_q4_0, f16_bits, f16_values, unrepack

RNG = np.random.default_rng(20260907)


# ---------------------------------------------------------------- generator

def test_splitmix64_published_outputs():
    # First outputs of splitmix64 from state 0 (Steele, Lea & Flood 2014;
    # the reference vectors used by SplittableRandom ports).
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F,
            0xF88BB8A8724C81EC]
    assert [synth.splitmix64_at(0, i) for i in range(4)] == want


def test_generator_counter_access_is_consistent():
    K = 96
    full = synth.q4_0_matrix(7, synth.weight_id(3), 20, K)
    part = synth.q4_0_rows(7, synth.weight_id(3), K, 5, 9)
    assert np.array_equal(full[5:14], part)
    lst = synth.q4_0_row_list(7, synth.weight_id(3), K, [19, 0, 11])
    assert np.array_equal(lst, full[[19, 0, 11]])
    a = synth.normal_f16(3, synth.act_id(1), 50)
    b = synth.normal_f16(3, synth.act_id(1), 20, i0=30)
    assert np.array_equal(a[30:], b)


def test_generator_distributions():
    g = synth.q4_0_matrix(synth.workload_seed(1), synth.weight_id(0), 512, 1024)
    blocks = g.reshape(-1, 18)
    d = f16_values(blocks[:, 0].astype(np.uint16) | (blocks[:, 1].astype(np.uint16) << 8))
    assert 0.0019 < np.abs(d).min() and np.abs(d).max() <= 0.05
    assert abs((d < 0).mean() - 0.5) < 0.01
    nib = np.concatenate([blocks[:, 2:] & 15, blocks[:, 2:] >> 4]).ravel()
    counts = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(counts - 1 / 16) < 0.002)
    x = f16_values(synth.normal_f16(synth.workload_seed(1), synth.act_id(0), 200000))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


# ---------------------------------------------------------------- f16 codecs

F16_TABLE = [  # (bits, value) from the IEEE-754 binary16 definition
    (0x0000, 0.0), (0x3C00, 1.0), (0xC000, -2.0), (0x7BFF, 65504.0),
    (0x0001, 2.0 ** -24), (0x03FF, 1023 * 2.0 ** -24), (0x0400, 2.0 ** -14),
    (0x3555, 0.333251953125), (0x3800, 0.5), (0x5640, 100.0),
    (0xFBFF, -65504.0), (0x8001, -(2.0 ** -24)),
]


def test_f16_decoder_table():
    for bits, val in F16_TABLE:
        assert oracle.f16_to_f64([bits])[0] == val
    assert math.copysign(1.0, oracle.f16_to_f64([0x8000])[0]) == -1.0
    assert oracle.f16_to_f64([0x7C00])[0] == math.inf
    assert oracle.f16_to_f64([0xFC00])[0] == -math.inf
    assert math.isnan(oracle.f16_to_f64([0x7E00])[0])


def test_f16_decoder_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


@pytest.mark.parametrize("encoder", ["synth", "oracle"])
def test_f16_encoders(encoder):
    enc = synth.f64_to_f16_bits if encoder == "synth" else oracle.f64_to_f16
    bits = np.arange(65536, dtype=np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(vals)
    # every finite f16 value encodes to itself
    assert np.array_equal(enc(vals[fin]), bits[fin])
    # midpoints between neighbours go to the even pattern
    pos = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2
    want = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint16)
    assert np.array_equal(enc(mid), want)
    assert np.array_equal(enc(-mid), want | 0x8000)
    # random doubles across the whole range against numpy's conversion
    r = np.concatenate([RNG.standard_normal(20000) * s for s in
                        (1e-7, 1e-5, 1e-3, 1.0, 100.0, 30000.0)])
    r = np.concatenate([r, [65519.99, 65520.0, 65536.0, 1e300, 2.0 ** -25,
                            3 * 2.0 ** -26, 1e-300, -0.0]])
    with np.errstate(over="ignore"):
        ref = r.astype(np.float16).view(np.uint16)
    assert np.array_equal(enc(r), ref)


# ---------------------------------------------------------------- GEMV pins

def _rand_codes(N, K):
    return RNG.integers(0, 16, size=(N, K))


def _rand_scales(N, K, lo=0.002, hi=0.05):
    mag = RNG.uniform(lo, hi, size=(N, K // 32)) * RNG.choice([-1, 1], size=(N, K // 32))
    return f16_bits(mag)


def test_all_codes_eight_give_zero():
    N, K = 7, 128
    rows = encode_q4_0(np.full((N, K), 8), _rand_scales(N, K))
    x = synth.activations(11, 3, K)
    y = oracle.q4_gemv(rows, K, x)
    assert np.array_equal(y, np.zeros_like(y))


def test_unit_vectors_pin_nibble_order_offset_and_scale():
    N, K = 5, 64
    q = _rand_codes(N, K)
    q[0, :16] = np.arange(16)            # every code appears
    d = _rand_scales(N, K)
    rows = encode_q4_0(q, d)
    dv = f16_values(d)
    for k in range(K):
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = 0x3C00                 # 1.0
        y = oracle.q4_gemv(rows, K, x)[0]
        want = (q[:, k] - 8) * dv[:, k // 32]
        assert np.array_equal(y, want), k
    # q = 0 -> -8d, q = 15 -> +7d
    x = np.zeros((1, K), dtype=np.uint16); x[0, 0] = 0x3C00
    assert oracle.q4_gemv(rows, K, x)[0][0] == -8 * dv[0, 0]
    x = np.zeros((1, K), dtype=np.uint16); x[0, 15] = 0x3C00
    assert oracle.q4_gemv(rows, K, x)[0][0] == 7 * dv[0, 0]


def test_single_nonzero_block():
    N, K = 4, 160
    q = np.full((N, K), 8)
    n0, b0 = 2, 3
    q[n0, 32 * b0: 32 * b0 + 32] = RNG.integers(0, 16, size=32)
    d = _rand_scales(N, K)
    rows = encode_q4_0(q, d)
    xi = RNG.integers(-3, 4, size=(1, K))             # small integers, exact in f16
    x = f16_bits(xi)
    y = oracle.q4_gemv(rows, K, x)[0]
    dot = int(np.dot(q[n0, 32 * b0: 32 * b0 + 32] - 8, xi[0, 32 * b0: 32 * b0 + 32]))
    assert y[n0] == dot * f16_values(d)[n0, b0]
    assert np.all(y[np.arange(N) != n0] == 0)


def test_linearity_in_scales():
    N, K = 6, 96
    q = _rand_codes(N, K)
    # scales with few significant bits so alpha*d1 + beta*d2 stays an f16
    d1 = RNG.integers(1, 32, size=(N, K // 32)) * 2.0 ** -10 * RNG.choice([-1, 1], size=(N, K // 32))
    d2 = RNG.integers(1, 32, size=(N, K // 32)) * 2.0 ** -10
    alpha, beta = 2.0, -0.5
    ds = alpha * d1 + beta * d2
    assert np.array_equal(f16_values(f16_bits(ds)), ds)
    x = synth.activations(5, 2, K)
    y1 = oracle.q4_gemv(encode_q4_0(q, f16_bits(d1)), K, x)
    y2 = oracle.q4_gemv(encode_q4_0(q, f16_bits(d2)), K, x)
    ys = oracle.q4_gemv(encode_q4_0(q, f16_bits(ds)), K, x)
    np.testing.assert_allclose(ys, alpha * y1 + beta * y2, rtol=1e-12, atol=1e-12)


def test_brute_force_exact_rationals():
    for (N, K) in [(3, 32), (2, 64), (4, 96)]:
        q = _rand_codes(N, K)
        d = _rand_scales(N, K)
        rows = encode_q4_0(q, d)
        x = synth.activations(17 + K, 2, K)
        y = oracle.q4_gemv(rows, K, x)
        xv = f16_values(x)
        dv = f16_values(d)
        for m in range(2):
            for n in range(N):
                exact = sum(Fraction(int(q[n, k]) - 8) * Fraction(dv[n, k // 32]) * Fraction(xv[m, k])
                            for k in range(K))
                assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)


def test_dense_matvec_equivalence_32x32_and_larger():
    for (N, K) in [(32, 32), (64, 256)]:
        q = _rand_codes(N, K)
        d = _rand_scales(N, K)
        W = (q - 8) * np.repeat(f16_values(d), 32, axis=1)
        x = synth.activations(3, 4, K)
        y = oracle.q4_gemv(encode_q4_0(q, d), K, x)
        ref = f16_values(x) @ W.T
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_threaded_rows_match_single_thread():
    N, K = 67, 256
    rows = synth.q4_0_matrix(9, synth.weight_id(0), N, K)
    x = synth.activations(9, 3, K)
    assert np.array_equal(oracle.q4_gemv(rows, K, x, threads=1),
                          oracle.q4_gemv(rows, K, x, threads=4))


# ---------------------------------------------------------------- golden fixture

def _load_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "q4_0_hand_cases.txt")
    cases = []
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        name, K, d, qs, x, y = [f.strip() for f in line.split("|")]
        cases.append((name, int(K), d, qs, x, float(y)))
    return cases


def golden_inputs(K, d, qs, x):
    nb = K // 32
    dl = [int(v, 16) for v in d.split()]
    ql = bytes.fromhex(qs.replace(" ", ""))
    assert len(dl) == nb and len(ql) == 16 * nb
    row = bytearray()
    for b in range(nb):
        row += bytes([dl[b] & 0xFF, dl[b] >> 8]) + ql[16 * b: 16 * b + 16]
    if x.startswith("ramp"):
        xs = [float(k) for k in range(K)]
    else:
        xs = [float(v) for v in x.split()]
        if len(xs) == 1:
            xs = xs * K
    return np.frombuffer(bytes(row), dtype=np.uint8), f16_bits(np.array(xs))[None, :]


def test_golden_hand_cases():
    for name, K, d, qs, x, y in _load_golden():
        rows, xb = golden_inputs(K, d, qs, x)
        assert oracle.q4_gemv(rows, K, xb)[0][0] == y, name


# ---------------------------------------------------------------- repack

@pytest.mark.parametrize("N,K", [(32, 32), (40, 64), (1, 96), (65, 160)])
def test_repack_round_trip_and_padding(N, K):
    g = synth.q4_0_matrix(21, synth.weight_id(1), N, K)
    p = oracle.repack(g, N, K)
    assert p.size == ((N + 31) // 32 * 32) * (K // 32) * 18
    back, pad = unrepack(p, N, K)
    assert np.array_equal(back, g)
    if pad.size:
        padb = pad.reshape(-1, K // 32, 18)
        assert np.all(padb[:, :, :2] == 0) and np.all(padb[:, :, 2:] == 0x88)


# ---------------------------------------------------------------- renorm and chain

def test_renorm_invariants():
    v = synth.normal_f16(1, synth.act_id(0), 5120)
    r = oracle.renorm(v)
    rv = f16_values(r)
    assert abs(np.sqrt(np.mean(rv ** 2)) - 1.0) < 1e-3
    # power-of-two scaling of the input leaves the output unchanged
    v4 = f16_bits(f16_values(v) * 4.0)
    assert np.array_equal(oracle.renorm(v4), r)
    # constant vectors map to +-1 exactly, zero to zero
    c = f16_bits(np.full(100, -3.25))
    assert np.array_equal(oracle.renorm(c), f16_bits(np.full(100, -1.0)))
    z = np.zeros(64, dtype=np.uint16)
    assert np.array_equal(oracle.renorm(z), z)
    # sign symmetry
    assert np.array_equal(oracle.renorm(v ^ 0x8000), r ^ 0x8000)


def test_unit_rms_scale_invariants():
    v = synth.normal_f16(2, synth.act_id(0), 4096)
    s = oracle.unit_rms_scale(v)
    # power-of-two scaling of the input divides the scale exactly
    assert oracle.unit_rms_scale(f16_bits(f16_values(v) * 8.0)) == s / 8.0
    # constant vectors: 1/|c|; zero: 0; sign-blind
    assert oracle.unit_rms_scale(f16_bits(np.full(37, -0.75))) == 1.0 / 0.75
    assert oracle.unit_rms_scale(np.zeros(9, dtype=np.uint16)) == 0.0
    assert oracle.unit_rms_scale(v ^ 0x8000) == s
    # renorm is the scaled vector rounded once
    assert np.array_equal(oracle.renorm(v), oracle.f64_to_f16(f16_values(v) * s))


def test_stack_scales_inputs_without_rounding():
    """One layer whose O matrix selects entry p[n] of its input with weight
    +-3/64: b[n] = f16(s * (+-3/64 * a[p[n]])) with a = f16(QKV x) and s its
    unit-RMS scale, rounded once (a second f16 rounding of s*a, before O,
    would change some entries)."""
    hidden, qkv_n, ffn = 64, 64, 64
    qkv = synth.q4_0_matrix(77, synth.weight_id(0), qkv_n, hidden)
    p_o = RNG.permutation(hidden); s_o = RNG.choice([-1, 1], hidden)
    o = signed_selection(hidden, hidden, p_o, s_o, d_bits=0x2A00)     # d = 3/64
    x = synth.normal_f16(77, synth.act_id(0), hidden)
    seen = {}
    oracle.stack_step(lambda l, t: {0: qkv, 1: o, 2: synth.q4_0_matrix(77, 3, 2 * ffn, hidden),
                                    3: synth.q4_0_matrix(77, 4, hidden, ffn)}[t],
                      x, 1, hidden, qkv_n, ffn, record=lambda i, xf, sc, y: seen.setdefault(i, (xf, sc, y)))
    a = oracle.f64_to_f16(oracle.q4_gemv(qkv, hidden, x[None, :])[0])
    s = oracle.unit_rms_scale(a)
    xf, sc, y = seen[1]
    assert np.array_equal(xf, a) and sc == s
    want = oracle.f64_to_f16(s * (s_o * 0.046875 * f16_values(a)[p_o]))
    assert np.array_equal(oracle.f64_to_f16(y), want)
    twice = oracle.f64_to_f16(s_o * 0.046875 * f16_values(oracle.f64_to_f16(s * f16_values(a)))[p_o])
    assert not np.array_equal(twice, want)


def signed_selection(N, K, src, sign, junk_from=None, d_bits=0x2800):
    """Q4_0 rows with one nonzero per row: row n = sign[n] * 2^-5 * e_{src[n]}
    (code 9 -> +d, code 7 -> -d, d = 2^-5).  Rows >= junk_from get random
    codes instead."""
    q = np.full((N, K), 8)
    q[np.arange(N), src] = np.where(sign > 0, 9, 7)
    if junk_from is not None:
        q[junk_from:] = RNG.integers(0, 16, size=(N - junk_from, K))
    d = np.full((N, K // 32), d_bits, dtype=np.uint16)
    return encode_q4_0(q, d)


def make_perm_stack(L, hidden, qkv_n, ffn):
    mats, maps = {}, []
    for l in range(L):
        p_qkv = RNG.permutation(hidden); s_qkv = RNG.choice([-1, 1], hidden)
        p_o = RNG.permutation(hidden); s_o = RNG.choice([-1, 1], hidden)
        p_gu = RNG.integers(0, hidden, ffn); s_gu = RNG.choice([-1, 1], ffn)
        p_dn = RNG.choice(ffn, hidden, replace=False); s_dn = RNG.choice([-1, 1], hidden)
        mats[(l, 0)] = signed_selection(qkv_n, hidden, np.concatenate([p_qkv, np.zeros(qkv_n - hidden, int)]),
                                        np.concatenate([s_qkv, np.ones(qkv_n - hidden, int)]), junk_from=hidden)
        mats[(l, 1)] = signed_selection(hidden, hidden, p_o, s_o)
        mats[(l, 2)] = signed_selection(2 * ffn, hidden, np.concatenate([p_gu, np.zeros(ffn, int)]),
                                        np.concatenate([s_gu, np.ones(ffn, int)]), junk_from=ffn)
        mats[(l, 3)] = signed_selection(hidden, ffn, p_dn, s_dn)
        maps.append([(p_qkv, s_qkv), (p_o, s_o), (p_gu, s_gu), (p_dn, s_dn)])
    return mats, maps


def perm_stack_expected(x_pm1, maps):
    v = x_pm1.copy()
    for layer in maps:
        for p, s in layer:
            v = s * v[p]
    return v


def test_stack_chain_closed_form():
    L, hidden, qkv_n, ffn = 3, 64, 96, 128
    mats, maps = make_perm_stack(L, hidden, qkv_n, ffn)
    x = RNG.choice([-1.0, 1.0], hidden)
    out = oracle.stack_step(lambda l, t: mats[(l, t)], f16_bits(x), L, hidden, qkv_n, ffn)
    assert np.array_equal(f16_values(out), perm_stack_expected(x, maps))


def make_gated_perm_stack(L, hidden, qkv_n, ffn):
    """Signed selections for every matrix, the up half of gate+up too."""
    mats, maps = {}, []
    for l in range(L):
        p_qkv = RNG.permutation(hidden); s_qkv = RNG.choice([-1, 1], hidden)
        p_o = RNG.permutation(hidden); s_o = RNG.choice([-1, 1], hidden)
        p_g = RNG.integers(0, hidden, ffn); s_g = RNG.choice([-1, 1], ffn)
        p_u = RNG.integers(0, hidden, ffn); s_u = RNG.choice([-1, 1], ffn)
        p_dn = RNG.choice(ffn, hidden, replace=False); s_dn = RNG.choice([-1, 1], hidden)
        mats[(l, 0)] = signed_selection(qkv_n, hidden, np.concatenate([p_qkv, np.zeros(qkv_n - hidden, int)]),
                                        np.concatenate([s_qkv, np.ones(qkv_n - hidden, int)]), junk_from=hidden)
        mats[(l, 1)] = signed_selection(hidden, hidden, p_o, s_o)
        mats[(l, 2)] = signed_selection(2 * ffn, hidden, np.concatenate([p_g, p_u]), np.concatenate([s_g, s_u]))
        mats[(l, 3)] = signed_selection(hidden, ffn, p_dn, s_dn)
        maps.append((p_qkv, s_qkv, p_o, s_o, p_g, s_g, p_u, s_u, p_dn, s_dn))
    return mats, maps


def test_gated_stack_chain_closed_form():
    """The gated chain on signed selections (row n of every matrix is
    +-2^-5 e_p(n)): each GEMV's output is f16(s * 2^-5 * sign * v[p]) for its
    input v and the input's unit-RMS scale s (1 for the step's own input),
    and the gated down GEMV's input is u = g/(1 + e^-g) * up of the f16
    gate and up halves, scaled by 1/sqrt(mean(u^2)).  Written here with
    numpy's exponential and sums, the oracle's with the C library's; f16
    rounding only where the chain rounds."""
    L, hidden, qkv_n, ffn = 2, 64, 96, 128
    mats, maps = make_gated_perm_stack(L, hidden, qkv_n, ffn)
    x = RNG.choice([-1.0, 1.0], hidden)
    out = oracle.stack_step(lambda l, t: mats[(l, t)], f16_bits(x), L, hidden, qkv_n, ffn, gated=True)

    def f16(v):
        return v.astype(np.float16).astype(np.float64)

    def scale(v):
        return 1.0 / np.sqrt(np.mean(v * v))

    v, s = x.copy(), 1.0
    for (p_qkv, s_qkv, p_o, s_o, p_g, s_g, p_u, s_u, p_dn, s_dn) in maps:
        a = f16(s * 2.0 ** -5 * s_qkv * v[p_qkv])         # QKV rows past hidden unused
        b = f16(scale(a) * 2.0 ** -5 * s_o * a[p_o])
        sb = scale(b)
        g = f16(sb * 2.0 ** -5 * s_g * b[p_g])
        up = f16(sb * 2.0 ** -5 * s_u * b[p_u])
        u = g / (1.0 + np.exp(-g)) * up
        v = f16(scale(u) * 2.0 ** -5 * s_dn * u[p_dn])
        s = scale(v)
    want = f16(s * v)
    assert np.array_equal(f16_values(out), want)


def test_gated_stack_differs_from_the_plain_chain_only_in_down():
    """gated=True changes the down GEMV's input and nothing before it: the
    first three GEMVs of each layer see the same inputs as in the plain
    chain (one layer), and the down input recorded is the whole gate+up
    output."""
    L, hidden, qkv_n, ffn = 1, 64, 96, 128
    mats, _ = make_gated_perm_stack(L, hidden, qkv_n, ffn)
    x = f16_bits(RNG.choice([-1.0, 1.0], hidden))
    rec_p, rec_g = {}, {}
    oracle.stack_step(lambda l, t: mats[(l, t)], x, L, hidden, qkv_n, ffn,
                      record=lambda i, xf, s, y: rec_p.setdefault(i, xf.copy()))
    oracle.stack_step(lambda l, t: mats[(l, t)], x, L, hidden, qkv_n, ffn, gated=True,
                      record=lambda i, xf, s, y: rec_g.setdefault(i, xf.copy()))
    for i in range(3):
        assert np.array_equal(rec_p[i], rec_g[i])
    assert rec_g[3].size == 2 * ffn and rec_p[3].size == ffn
    assert np.array_equal(rec_g[3][:ffn], rec_p[3])
