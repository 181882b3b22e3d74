"""Q8_0 GEMV parity through the C ABI (q4gemv_q8_0_*), against the fp64
oracle on the same seeded inputs."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, bits_of, f16_dev, rel_err

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


def packed_q8(eng, gguf, N, K):
    return eng.repack_q8_0(torch.from_numpy(np.ascontiguousarray(gguf).reshape(-1)).cuda(), N, K)


def q8_case(eng, N, K, M, seed, tid=0):
    gguf = synth.q8_0_matrix(seed, synth.weight_id(tid), N, K)
    x = synth.activations(seed, M, K)
    W = packed_q8(eng, gguf, N, K)
    y = eng.run_q8_0(W, f16_dev(x).reshape(M, K), N, K)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return gguf, x, bits_of(y)


@pytest.mark.parametrize("N,K", [(1, 32), (33, 64), (257, 160), (1024, 1024), (40, 6400)])
def test_q8_repack_bit_exact(eng, N, K):
    gguf = synth.q8_0_matrix(21, synth.weight_id(1), N, K)
    got = packed_q8(eng, gguf, N, K).cpu().numpy()
    assert np.array_equal(got, oracle.repack_q8(gguf, N, K))


@pytest.mark.parametrize("N,K", [(1024, 1024), (5120, 5120), (34816, 5120), (5120, 17408)])
def test_q8_gemv_m1_config_shapes(eng, N, K):
    gguf, x, y = q8_case(eng, N, K, 1, synth.workload_seed(1) + 80)
    ref = oracle.q8_gemv(gguf, K, x, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= TOL, err


@pytest.mark.parametrize("N,K", [(1, 32), (31, 32), (33, 64), (257, 160), (4096, 64), (100, 96)])
@pytest.mark.parametrize("M", [1, 2])
def test_q8_gemv_edge_shapes(eng, M, N, K):
    gguf, x, y = q8_case(eng, N, K, M, 700 + N + K + M)
    ref = oracle.q8_gemv(gguf, K, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


def test_q8_gemv_m2_gate_up(eng):
    gguf, x, y = q8_case(eng, 34816, 5120, 2, 91)
    ref = oracle.q8_gemv(gguf, 5120, x, threads=THREADS)
    assert rel_err(y, ref) <= TOL


def test_q8_extreme_codes_and_special_inputs(eng):
    """Codes -128 and 127 everywhere with the largest scales, then a NaN in x:
    exact where representable, NaN outputs for a non-finite input."""
    N, K = 64, 256
    g = synth.q8_0_matrix(5, synth.weight_id(2), N, K).reshape(N, K // 32, 34)
    g[:, :, 2:] = np.where(np.arange(32) % 2 == 0, 0x80, 0x7F).astype(np.uint8)   # -128, 127
    g = g.reshape(N, -1)
    x = synth.activations(5, 1, K)
    W = packed_q8(eng, g, N, K)
    y = bits_of(eng.run_q8_0(W, f16_dev(x), N, K))
    assert rel_err(y, oracle.q8_gemv(g, K, x)) <= TOL
    xn = x.copy()
    xn[0, 5] = 0x7E00                                 # NaN
    y = bits_of(eng.run_q8_0(W, f16_dev(xn), N, K)).view(np.float16)
    assert np.all(np.isnan(y.astype(np.float64)))


def test_q8_deterministic(eng):
    N, K = 5120, 5120
    gguf = synth.q8_0_matrix(6, synth.weight_id(0), N, K)
    x = f16_dev(synth.activations(6, 1, K))
    W = packed_q8(eng, gguf, N, K)
    a = bits_of(eng.run_q8_0(W, x, N, K))
    b = bits_of(eng.run_q8_0(W, x, N, K))
    assert np.array_equal(a, b)


def test_q8_validate_limits(eng):
    A = 1 << 20
    assert q4.q4gemv_q8_0_validate(3, 32, 32, A, A, A) == q4.Q4_OK          # tensor-core GEMM
    assert q4.q4gemv_q8_0_validate(256, 32, 32, A, A, A) == q4.Q4_OK
    assert q4.q4gemv_q8_0_validate(1, 32, 65536, A, A, A) == q4.Q4_OK      # wide K: GEMM path
    assert q4.q4gemv_q8_0_validate(0, 32, 32, A, A, A) == q4.Q4_EUNSUPPORTED
    assert q4.q4gemv_q8_0_validate(257, 32, 32, A, A, A) == q4.Q4_EUNSUPPORTED
    assert q4.q4gemv_q8_0_validate(1, 32, 48, A, A, A) == q4.Q4_ESHAPE
    assert q4.q4gemv_q8_0_validate(1, 32, 32, A + 8, A, A) == q4.Q4_EALIGN


# ---------------------------------------------------------------- M >= 3 (and wide K): tensor cores
# (mma.sync kernel up to M = 16, the tcgen05 GEMM beyond)

@pytest.mark.parametrize("N,K,M", [(256, 64, 3), (300, 96, 4), (520, 160, 16), (33, 1056, 17),
                                   (1024, 1024, 86), (5, 32, 256), (2048, 5120, 169),
                                   (96, 65536, 1), (40, 40960, 2)])
def test_q8_gemm_shapes_full(eng, N, K, M):
    gguf, x, y = q8_case(eng, N, K, M, 1300 + N + K + M)
    ref = oracle.q8_gemv(gguf, K, x, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= 5.2e-4, err            # exact two-part weights: output rounding only


@pytest.mark.parametrize("M", [16, 169])
@pytest.mark.parametrize("N,K", [(34816, 5120), (5120, 17408)])
def test_q8_gemm_full_shapes_sampled(eng, M, N, K):
    gguf, x, y = q8_case(eng, N, K, M, synth.workload_seed(3) + 2000 + M, tid=0 if K == 5120 else 1)
    y = y.reshape(M, N)
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(N, 160, replace=False), [0, 255, 256, N - 1]]))
    ref = oracle.q8_gemv(np.ascontiguousarray(gguf[rows]), K, x, threads=THREADS)
    assert rel_err(np.ascontiguousarray(y[:, rows]), ref) <= TOL


@pytest.mark.parametrize("M", [4, 16, 40])
def test_q8_gemm_extreme_codes_and_deterministic(eng, M):
    N, K = 300, 512
    g = synth.q8_0_matrix(15, synth.weight_id(2), N, K).reshape(N, K // 32, 34)
    g[:, :, 2:] = np.where(np.arange(32) % 3 == 0, 0x80, np.where(np.arange(32) % 3 == 1, 0x7F, 0xFF))
    g = g.reshape(N, -1)
    x = synth.activations(15, M, K)
    W = packed_q8(eng, g, N, K)
    xd = f16_dev(x).reshape(M, K)
    a = bits_of(eng.run_q8_0(W, xd, N, K))
    b = bits_of(eng.run_q8_0(W, xd, N, K))
    assert np.array_equal(a, b)
    assert rel_err(a, oracle.q8_gemv(g, K, x)) <= 5.2e-4
