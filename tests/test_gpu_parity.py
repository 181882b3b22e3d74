"""GPU parity: the CUDA path through the C-ABI against the fp64 oracle on the
same seeded inputs (repack bit-exact, GEMV within TOL, the decode-step chain
end to end and teacher-forced per GEMV)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, bits_of, f16_dev, packed_on_gpu, rel_err, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import q4_quantized_decode_b200 as q4  # noqa: E402

THREADS = 8


@pytest.fixture(scope="module")
def eng():
    e = q4.Q4Gemv(0)
    yield e
    e.close()


def gemv_case(eng, N, K, M, seed, tid=0, x=None):
    gguf = synth.q4_0_matrix(seed, synth.weight_id(tid), N, K)
    if x is None:
        x = synth.activations(seed, M, K)
    W = packed_on_gpu(eng, gguf, N, K)
    y = eng.run(W, f16_dev(x).reshape(M, K), N, K)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return gguf, x, bits_of(y)


# ---------------------------------------------------------------- repack

@pytest.mark.parametrize("N,K", [(1, 32), (33, 64), (64, 1024), (100, 96), (5120, 5120),
                                 (1000, 17408)])
def test_repack_bit_exact(eng, N, K):
    gguf = synth.q4_0_matrix(77, synth.weight_id(2), N, K)
    p = packed_on_gpu(eng, gguf, N, K).cpu().numpy()
    assert np.array_equal(p, oracle.repack(gguf, N, K))


# ---------------------------------------------------------------- GEMV, M = 1, 2

M1_SHAPES = {
    "gemv_1024x1024": (1024, 1024, 0),
    "qkv_7168x5120": (7168, 5120, 4),
    "o_5120x5120": (5120, 5120, 1),
    "gate_up_34816x5120": (34816, 5120, 2),
    "down_5120x17408": (5120, 17408, 2),
}


@pytest.mark.parametrize("name", list(M1_SHAPES))
def test_gemv_m1_shapes(eng, name):
    N, K, c = M1_SHAPES[name]
    gguf, x, y = gemv_case(eng, N, K, 1, synth.workload_seed(c), tid=0 if "down" not in name else 1)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= TOL, err


@pytest.mark.parametrize("N,K", [(1024, 1024), (5120, 17408), (300, 5120)])
def test_gemv_m2(eng, N, K):
    gguf, x, y = gemv_case(eng, N, K, 2, 91)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("M", [4, 16])
@pytest.mark.parametrize("N,K", [(34816, 5120), (5120, 17408)])
def test_gemv_small_m_shapes(eng, M, N, K):
    """Speculative-verify batch (M=4) and prefill chunk (M=16) on the FFN shapes."""
    gguf, x, y = gemv_case(eng, N, K, M, synth.workload_seed(3) + M, tid=0 if K == 5120 else 1)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= TOL, err


@pytest.mark.parametrize("M", [3, 5, 8, 9, 13, 16])
@pytest.mark.parametrize("N,K", [(1, 32), (33, 64), (100, 96), (257, 160), (4096, 64), (40, 6400),
                                 (64, 40960)])
def test_gemv_small_m_edge_shapes(eng, M, N, K):
    gguf, x, y = gemv_case(eng, N, K, M, 500 + 7 * M + N + K)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("M", [1, 2])
def test_gemv_wide_k_uses_tensor_core_path(eng, M):
    """K beyond the shared-memory limit of the M <= 2 kernel."""
    N, K = 96, 65536
    gguf, x, y = gemv_case(eng, N, K, M, 4242)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("N,K", [(1, 32), (31, 32), (33, 64), (100, 96), (7, 1056), (257, 160),
                                 (8192, 32), (4096, 64), (2, 17408), (40, 40960)])
def test_gemv_edge_shapes(eng, N, K):
    gguf, x, y = gemv_case(eng, N, K, 1, 1000 + N + K)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


def test_all_codes_eight_give_exact_zero(eng):
    N, K = 96, 256
    gguf = synth.q4_0_matrix(5, synth.weight_id(0), N, K).reshape(N, K // 32, 18)
    gguf[:, :, 2:] = 0x88
    x = synth.activations(5, 1, K)
    W = packed_on_gpu(eng, gguf.reshape(N, -1), N, K)
    y = bits_of(eng.run(W, f16_dev(x), N, K))
    assert np.all((y & 0x7FFF) == 0)


def test_zero_and_tiny_activation_blocks(eng):
    N, K = 64, 256
    gguf = synth.q4_0_matrix(6, synth.weight_id(0), N, K)
    x = synth.activations(6, 1, K)
    x[0, 0:32] = 0                                        # an all-zero block
    x[0, 32:64] = synth.f64_to_f16_bits(np.linspace(-3e-6, 3e-6, 32))   # subnormals
    x[0, 64:96] = synth.f64_to_f16_bits(np.linspace(-60000, 60000, 32) / 1000)
    W = packed_on_gpu(eng, gguf, N, K)
    y = bits_of(eng.run(W, f16_dev(x), N, K))
    ref = oracle.q4_gemv(gguf, K, x)
    assert rel_err(y, ref) <= TOL


def outlier_x(seed, M, K):
    """Activations whose every other 32-entry block holds one entry 2^12 (or
    more) times the largest of the others, at a position that moves across
    the lane groups: the blocks where the int16 conversion rounds the small
    entries (to 2^-15 of the block maximum) instead of holding them exactly."""
    # Base entries scaled by 2^-5 (exact) so the outputs stay inside the
    # binary16 range with an outlier in every other block.
    x = synth.activations(seed, M, K).view(np.float16).astype(np.float64) / 32.0
    for m in range(M):
        for b in range(0, K // 32, 2):
            blk = x[m, 32 * b:32 * b + 32]
            p = (7 * b + 3 * m) % 32
            others = np.delete(np.abs(blk), p)
            blk[p] = (1 if (b + m) % 4 < 2 else -1) * 4096.0 * max(float(others.max()), 2.0 ** -10)
    xb = synth.f64_to_f16_bits(x.reshape(-1)).reshape(M, K)
    v = xb.view(np.float16).astype(np.float64)
    for m in range(M):
        for b in range(0, K // 32, 2):
            blk = np.abs(v[m, 32 * b:32 * b + 32])
            assert blk.max() >= 4096 * np.sort(blk)[-2]
    return xb


@pytest.mark.parametrize("M,N,K", [(1, 1024, 1024), (1, 5120, 17408), (2, 300, 5120), (2, 4096, 1024)])
def test_same_block_outlier_activations(eng, M, N, K):
    gguf = synth.q4_0_matrix(71, synth.weight_id(1), N, K)
    x = outlier_x(71 + K, M, K)
    W = packed_on_gpu(eng, gguf, N, K)
    y = bits_of(eng.run(W, f16_dev(x).reshape(M, K), N, K))
    assert eng.sync_status() == q4.Q4_OK
    err = rel_err(y, oracle.q4_gemv(gguf, K, x, threads=THREADS))
    assert err <= TOL, err


def test_nan_activation_gives_nan(eng):
    N, K = 64, 128
    gguf = synth.q4_0_matrix(8, synth.weight_id(0), N, K)
    x = synth.activations(8, 1, K)
    x[0, 40] = 0x7E00
    W = packed_on_gpu(eng, gguf, N, K)
    y = bits_of(eng.run(W, f16_dev(x), N, K)).view(np.float16)
    ref = oracle.q4_gemv(gguf, K, x)
    assert np.all(np.isnan(ref)) and np.all(np.isnan(y))


def test_overflow_gives_signed_inf(eng):
    N, K = 32, 64
    from tests.q4_helpers import encode_q4_0, f16_bits
    q = np.full((N, K), 15)
    q[N // 2:] = 0
    d = f16_bits(np.full((N, K // 32), 0.05))
    gguf = encode_q4_0(q, d)
    x = f16_bits(np.full((1, K), 60000.0))
    W = packed_on_gpu(eng, gguf, N, K)
    y = bits_of(eng.run(W, f16_dev(x), N, K)).view(np.float16).astype(np.float64)[0]
    ref = oracle.q4_gemv(gguf, K, x)[0]
    assert np.all(np.abs(ref) > 65520)
    assert np.array_equal(y, np.where(ref > 0, np.inf, -np.inf))


def test_deterministic_bits(eng):
    N, K = 5120, 17408
    gguf = synth.q4_0_matrix(3, synth.weight_id(0), N, K)
    x = synth.activations(3, 1, K)
    W = packed_on_gpu(eng, gguf, N, K)
    xd = f16_dev(x)
    y1 = bits_of(eng.run(W, xd, N, K))
    y2 = bits_of(eng.run(W, xd, N, K))
    assert np.array_equal(y1, y2)


def test_user_stream_capture_of_run(eng):
    N, K = 2048, 5120
    gguf = synth.q4_0_matrix(4, synth.weight_id(0), N, K)
    x = synth.activations(4, 1, K)
    W = packed_on_gpu(eng, gguf, N, K)
    xd = f16_dev(x)
    y = torch.empty(1, N, dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        eng.run(W, xd, N, K, out=y)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert rel_err(bits_of(y), oracle.q4_gemv(gguf, K, x, threads=THREADS)) <= TOL


# ---------------------------------------------------------------- decode-step chain

def build_stack(eng, L, hidden, qkv_n, ffn, seed):
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    layers, ggufs = [], {}
    for l in range(L):
        mats = []
        for t, (N, K) in enumerate(dims):
            g = synth.q4_0_matrix(seed, synth.weight_id(4 * l + t), N, K)
            ggufs[(l, t)] = g
            mats.append(packed_on_gpu(eng, g, N, K))
        layers.append(tuple(mats))
    return layers, ggufs


def run_stack_traced(eng, layers, x, hidden, qkv_n, ffn):
    L = len(layers)
    kx, ky = q4.stack_trace_dims(hidden, qkv_n, ffn)
    tx = torch.zeros(4 * L, kx, dtype=torch.float16, device="cuda")
    ty = torch.zeros(4 * L, ky, dtype=torch.float16, device="cuda")
    out = eng.run_stack(layers, f16_dev(x), hidden, qkv_n, ffn, trace_x=tx, trace_y=ty)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return bits_of(out), bits_of(tx), bits_of(ty)


def check_teacher_forced(ggufs, x_in, tx, ty, L, hidden, qkv_n, ffn, rows=None, seed=0):
    """Each GEMV i recomputed by the oracle from the GPU's own input: the
    traced f16 vector (x_in, then the previous output's first K entries,
    checked bit for bit) times its unit-RMS scale, taken in fp64 here (the
    GPU's fp32 scale is a few ulp away, far inside the tolerance)."""
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    rng = np.random.default_rng(seed)
    worst = 0.0
    for i in range(4 * L):
        l, t = divmod(i, 4)
        N, K = dims[t]
        xin = tx[i, :K]
        if i == 0:
            assert np.array_equal(xin, x_in)
            s = 1.0
        else:
            assert np.array_equal(xin, ty[i - 1, :K]), i
            s = oracle.unit_rms_scale(xin)
        g = ggufs(l, t) if callable(ggufs) else ggufs[(l, t)]
        if rows is None:
            ref = s * oracle.q4_gemv(g, K, xin[None, :], threads=THREADS)[0]
            got = ty[i, :N]
        else:
            sel = np.sort(rng.choice(N, size=min(rows, N), replace=False))
            ref = s * oracle.q4_gemv(g(sel) if callable(g) else g[sel], K, xin[None, :])[0]
            got = ty[i, sel]
            # rms(y) from the GPU output itself for the error denominator
            rms = np.sqrt(np.mean(ty[i, :N].view(np.float16).astype(np.float64) ** 2))
            den = np.maximum(np.abs(ref), rms)
            gv = got.view(np.float16).astype(np.float64)
            if not np.all(np.isfinite(gv)):
                return float("inf")
            e = float(np.max(np.abs(gv - ref) / den))
            worst = max(worst, e)
            continue
        worst = max(worst, rel_err(got, ref))
    return worst


def test_stack_small_end_to_end_and_teacher_forced(eng):
    L, hidden, qkv_n, ffn = 2, 256, 384, 512
    layers, ggufs = build_stack(eng, L, hidden, qkv_n, ffn, 4321)
    x = synth.normal_f16(4321, synth.act_id(0), hidden)
    out, tx, ty = run_stack_traced(eng, layers, x, hidden, qkv_n, ffn)
    assert check_teacher_forced(ggufs, x, tx, ty, L, hidden, qkv_n, ffn) <= TOL
    # End to end, two layers (eight GEMVs) stay within the GEMV tolerance: an
    # ideal fp32 kernel reproduces the oracle here to 4e-6
    # (tests/test_chain_drift_cpu.py); drift past 2e-3 needs longer chains.
    want = oracle.stack_step(lambda l, t: ggufs[(l, t)], x, L, hidden, qkv_n, ffn)
    drift = rel_err(out, oracle.f16_to_f64(want))
    print(f"end-to-end drift after {L} layers: {drift:.2e}")
    assert drift <= TOL, drift
    # final renorm of the GPU's own last output
    assert np.abs(oracle.renorm(ty[4 * L - 1, :hidden]).astype(np.int32) - out.astype(np.int32)).max() <= 1
    # without traces the same bits come out
    out2 = bits_of(eng.run_stack(layers, f16_dev(x), hidden, qkv_n, ffn))
    assert np.array_equal(out, out2)


def test_stack_host_vectors(eng):
    """x_in / x_out in host memory (pinned or pageable) give the same bits as
    device vectors; the copies happen inside the call."""
    L, hidden, qkv_n, ffn = 1, 256, 384, 512
    layers, _ = build_stack(eng, L, hidden, qkv_n, ffn, 99)
    x = synth.normal_f16(99, synth.act_id(0), hidden)
    want = bits_of(eng.run_stack(layers, f16_dev(x), hidden, qkv_n, ffn))
    for pinned in (True, False):
        xh = torch.from_numpy(x.view(np.float16).copy())
        oh = torch.empty(hidden, dtype=torch.float16)
        if pinned:
            xh, oh = xh.pin_memory(), oh.pin_memory()
        eng.run_stack(layers, xh, hidden, qkv_n, ffn, x_out=oh)
        torch.cuda.synchronize()
        assert eng.sync_status() == q4.Q4_OK
        assert np.array_equal(oh.numpy().view(np.uint16), want), pinned
    # host in, device out
    od = torch.empty(hidden, dtype=torch.float16, device="cuda")
    eng.run_stack(layers, torch.from_numpy(x.view(np.float16).copy()), hidden, qkv_n, ffn, x_out=od)
    assert np.array_equal(bits_of(od), want)


def test_stack_outlier_input_teacher_forced(eng):
    """The step's first GEMV converts x_in itself: same-block outliers there."""
    L, hidden, qkv_n, ffn = 1, 512, 640, 768
    layers, ggufs = build_stack(eng, L, hidden, qkv_n, ffn, 808)
    x = outlier_x(808, 1, hidden)[0]
    out, tx, ty = run_stack_traced(eng, layers, x, hidden, qkv_n, ffn)
    assert check_teacher_forced(ggufs, x, tx, ty, L, hidden, qkv_n, ffn) <= TOL


def test_device_wait_timeout_is_reported_and_recoverable():
    """A bounded device wait that runs out: the step's first inter-GEMV wait
    is given an unreachable condition and a short poll budget (the "timeout"
    test knob).  The kernel must return (the stream synchronises), the error
    word must read Q4_ETIMEOUT, and the next call on the same handle must
    run normally and give the right result."""
    eng = q4.Q4Gemv(0)
    L, hidden, qkv_n, ffn = 1, 256, 384, 512
    layers, ggufs = build_stack(eng, L, hidden, qkv_n, ffn, 31)
    x = synth.normal_f16(31, synth.act_id(0), hidden)
    xd = f16_dev(x)
    want = bits_of(eng.run_stack(layers, xd, hidden, qkv_n, ffn))
    assert eng.sync_status() == q4.Q4_OK
    eng.set_fault("timeout")
    out = torch.zeros(hidden, dtype=torch.float16, device="cuda")
    eng.run_stack(layers, xd, hidden, qkv_n, ffn, x_out=out)
    torch.cuda.synchronize()                      # the kernel gave up and returned
    assert eng.sync_status() == q4.Q4_ETIMEOUT
    assert eng.sync_status() == q4.Q4_OK          # the word was cleared
    eng.set_fault("none")
    got = bits_of(eng.run_stack(layers, xd, hidden, qkv_n, ffn, x_out=out))
    assert eng.sync_status() == q4.Q4_OK
    assert np.array_equal(got, want)
    ref = oracle.stack_step(lambda l, t: ggufs[(l, t)], x, L, hidden, qkv_n, ffn)
    assert rel_err(got, oracle.f16_to_f64(ref)) <= TOL
    eng.close()


def test_stack_signed_permutation_closed_form(eng):
    from tests.test_oracle_pins import make_perm_stack, perm_stack_expected
    L, hidden, qkv_n, ffn = 3, 64, 96, 128
    mats, maps = make_perm_stack(L, hidden, qkv_n, ffn)
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    layers = [tuple(packed_on_gpu(eng, mats[(l, t)], *dims[t]) for t in range(4)) for l in range(L)]
    x = np.random.default_rng(1).choice([-1.0, 1.0], hidden)
    xb = synth.f64_to_f16_bits(x)
    out = bits_of(eng.run_stack(layers, f16_dev(xb), hidden, qkv_n, ffn))
    want = perm_stack_expected(x, maps)
    assert np.array_equal(out.view(np.float16).astype(np.float64), want)


def test_stack_graph_replay_follows_input(eng):
    L, hidden, qkv_n, ffn = 1, 128, 192, 256
    layers, ggufs = build_stack(eng, L, hidden, qkv_n, ffn, 55)
    xa = synth.normal_f16(55, synth.act_id(0), hidden)
    xb = synth.normal_f16(55, synth.act_id(1), hidden)
    xin = f16_dev(xa)
    xout = torch.empty(hidden, dtype=torch.float16, device="cuda")
    eng.run_stack(layers, xin, hidden, qkv_n, ffn, x_out=xout)
    oa = bits_of(xout)
    xin.copy_(f16_dev(xb))                        # same pointers: graph replay
    eng.run_stack(layers, xin, hidden, qkv_n, ffn, x_out=xout)
    ob = bits_of(xout)
    wa = oracle.stack_step(lambda l, t: ggufs[(l, t)], xa, L, hidden, qkv_n, ffn)
    wb = oracle.stack_step(lambda l, t: ggufs[(l, t)], xb, L, hidden, qkv_n, ffn)
    assert rel_err(oa, oracle.f16_to_f64(wa)) <= TOL
    assert rel_err(ob, oracle.f16_to_f64(wb)) <= TOL
    assert not np.array_equal(oa, ob)
    # x_out aliasing x_in is allowed
    eng.run_stack(layers, xin, hidden, qkv_n, ffn, x_out=xin)
    assert np.array_equal(bits_of(xin), ob)


def test_stack_persistent_matches_per_gemv_kernels(monkeypatch):
    """The one-launch step and the graph of per-GEMV kernels run the same
    per-warp arithmetic over the same split: identical bits at full width."""
    L, hidden, qkv_n, ffn = 2, 5120, 7168, 17408
    outs = {}
    for mode in ("persistent", "kernels"):
        monkeypatch.setenv("Q4GEMV_STACK_MODE", mode)
        e = q4.Q4Gemv(0)
        if mode == "persistent":
            layers, _ = build_stack(e, L, hidden, qkv_n, ffn, 77)
        x = synth.normal_f16(77, synth.act_id(0), hidden)
        o1, tx, ty = run_stack_traced(e, layers, x, hidden, qkv_n, ffn)
        outs[mode] = (o1, tx, ty)
        e.close()
    for a, b in zip(outs["persistent"], outs["kernels"]):
        assert np.array_equal(a, b)


@pytest.mark.slow
def test_stack_full_27b_teacher_forced_sampled():
    """The full 64-layer, 27B-shaped step (11.9 GB of Q4_0), checked per GEMV
    on sampled rows from the GPU's own traced inputs."""
    eng = q4.Q4Gemv(0)
    L, hidden, qkv_n, ffn = 64, 5120, 7168, 17408
    seed = synth.workload_seed(4)
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    layers = []
    for l in range(L):
        layers.append(tuple(packed_on_gpu(eng, synth.q4_0_matrix(seed, synth.weight_id(4 * l + t), *dims[t]),
                                          *dims[t]) for t in range(4)))
    x = synth.normal_f16(seed, synth.act_id(0), hidden)
    out, tx, ty = run_stack_traced(eng, layers, x, hidden, qkv_n, ffn)

    def rows_of(l, t):
        K = dims[t][1]
        return lambda sel: synth.q4_0_row_list(seed, synth.weight_id(4 * l + t), K, sel)

    worst = check_teacher_forced(rows_of, x, tx, ty, L, hidden, qkv_n, ffn, rows=24, seed=9)
    assert worst <= TOL, worst
    # The first and the last layer in full: every row of all four GEMVs
    # (the CTA-boundary tiles, the ragged QKV tail and the pre-converted
    # hand-off are all exercised at full width).
    for l in (0, L - 1):
        for t, (N, K) in enumerate(dims):
            i = 4 * l + t
            xin = tx[i, :K]
            if i > 0:
                assert np.array_equal(xin, ty[i - 1, :K]), i
            s = 1.0 if i == 0 else oracle.unit_rms_scale(xin)
            g = synth.q4_0_matrix(seed, synth.weight_id(i), N, K)
            ref = s * oracle.q4_gemv(g, K, xin[None, :], threads=THREADS)[0]
            err = rel_err(ty[i, :N], ref)
            assert err <= TOL, (l, t, err)
    assert np.abs(oracle.renorm(ty[4 * L - 1, :hidden]).astype(np.int32) - out.astype(np.int32)).max() <= 1
    del layers
    eng.close()


# ---------------------------------------------------------------- host failures

def test_fault_injection_and_invalid_calls(eng):
    N, K = 64, 64
    gguf = synth.q4_0_matrix(1, synth.weight_id(0), N, K)
    W = packed_on_gpu(eng, gguf, N, K)
    x = f16_dev(synth.activations(1, 1, K))
    y = torch.full((1, N), 7.0, dtype=torch.float16, device="cuda")
    h, st = eng.h, q4._stream(None)
    eng.set_fault("launch")
    assert q4.q4gemv_run(h, W.data_ptr(), x.data_ptr(), y.data_ptr(), 1, N, K, st) == q4.Q4_EFAULTINJ
    eng.set_fault("none")
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)                     # nothing was launched
    assert q4.q4gemv_run(h, W.data_ptr() + 8, x.data_ptr(), y.data_ptr(), 1, N, K, st) == q4.Q4_EALIGN
    assert q4.q4gemv_run(h, W.data_ptr(), x.data_ptr(), y.data_ptr(), 1, N, 48, st) == q4.Q4_ESHAPE
    assert q4.q4gemv_run(h, W.data_ptr(), x.data_ptr(), y.data_ptr(), 0, N, K, st) == q4.Q4_EUNSUPPORTED
    assert "M=0" in q4.q4gemv_last_error(h)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    # graph and allocation faults in the decode-step runner
    L, hidden, qkv_n, ffn = 1, 64, 96, 128
    layers, _ = build_stack(eng, L, hidden, qkv_n, ffn, 2)
    xs = f16_dev(synth.normal_f16(2, synth.act_id(0), hidden))
    fresh = q4.Q4Gemv(0)
    fresh.set_fault("alloc")
    with pytest.raises(q4.Q4Error) as e:
        fresh.run_stack(layers, xs, hidden, qkv_n, ffn)
    assert e.value.status == q4.Q4_EFAULTINJ
    fresh.set_fault("launch")
    with pytest.raises(q4.Q4Error) as e:
        fresh.run_stack(layers, xs, hidden, qkv_n, ffn)
    assert e.value.status == q4.Q4_EFAULTINJ
    fresh.set_fault("none")
    fresh.run_stack(layers, xs, hidden, qkv_n, ffn)
    assert fresh.sync_status() == q4.Q4_OK
    fresh.close()
    eng.run(W, x, N, K)
    assert eng.sync_status() == q4.Q4_OK


def test_graph_fault_in_per_gemv_mode(monkeypatch):
    monkeypatch.setenv("Q4GEMV_STACK_MODE", "kernels")
    eng = q4.Q4Gemv(0)
    L, hidden, qkv_n, ffn = 1, 64, 96, 128
    layers, _ = build_stack(eng, L, hidden, qkv_n, ffn, 3)
    xs = f16_dev(synth.normal_f16(3, synth.act_id(0), hidden))
    eng.set_fault("graph")
    with pytest.raises(q4.Q4Error) as e:
        eng.run_stack(layers, xs, hidden, qkv_n, ffn)
    assert e.value.status == q4.Q4_EFAULTINJ
    eng.set_fault("none")
    eng.run_stack(layers, xs, hidden, qkv_n, ffn)
    assert eng.sync_status() == q4.Q4_OK
    eng.close()


def test_create_fault_from_environment(monkeypatch):
    monkeypatch.setenv("Q4GEMV_FAULT", "alloc")
    st, h = q4.q4gemv_create(0)
    assert st == q4.Q4_EFAULTINJ and not h.value
