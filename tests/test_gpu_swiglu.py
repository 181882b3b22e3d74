"""The down GEMV fed directly by the gate+up GEMV (q4gemv_run_swiglu):
y = W (SiLU(gate) * up) through the C ABI against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, bits_of, f16_dev, packed_on_gpu, rel_err

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


def swiglu_case(eng, rows, gu, N, K):
    W = packed_on_gpu(eng, rows, N, K)
    y = eng.run_swiglu(W, f16_dev(gu).reshape(-1), N, K)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return bits_of(y)


@pytest.mark.parametrize("N,K", [(5120, 17408), (1, 32), (33, 64), (257, 160), (40, 6400),
                                 (4096, 1024)])
def test_swiglu_gemv_shapes(eng, N, K):
    rows = synth.q4_0_matrix(600 + N, synth.weight_id(1), N, K)
    gu = synth.activations(601 + K, 1, 2 * K)
    y = swiglu_case(eng, rows, gu, N, K)
    ref = oracle.q4_gemv_swiglu(rows, K, gu, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= TOL, err


def test_ffn_pair_teacher_forced(eng):
    """gate+up GEMV (34816 x 5120) on the GPU, then the gated down GEMV
    (5120 x 17408) on the GPU's own gate+up output."""
    H, F = 5120, 17408
    seed = synth.workload_seed(2) + 500
    gu_rows = synth.q4_0_matrix(seed, synth.weight_id(0), 2 * F, H)
    dn_rows = synth.q4_0_matrix(seed, synth.weight_id(1), H, F)
    x = synth.activations(seed, 1, H)
    Wgu = packed_on_gpu(eng, gu_rows, 2 * F, H)
    Wdn = packed_on_gpu(eng, dn_rows, H, F)
    g = eng.run(Wgu, f16_dev(x), 2 * F, H)
    y = eng.run_swiglu(Wdn, g.reshape(-1), H, F)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    gb = bits_of(g).reshape(1, -1)
    # the first GEMV against the oracle, then the second from its output
    rows = np.random.default_rng(0).choice(2 * F, 256, replace=False)
    assert rel_err(gb[:, rows], oracle.q4_gemv(gu_rows[rows], H, x)) <= TOL
    ref = oracle.q4_gemv_swiglu(dn_rows, F, gb, threads=THREADS)
    assert rel_err(bits_of(y), ref) <= TOL


def test_saturated_gates(eng):
    """Gates deep in both tails (|g| = 12..30): SiLU is the identity or
    vanishes; zero up halves give zero outputs."""
    N, K = 64, 512
    rows = synth.q4_0_matrix(77, synth.weight_id(2), N, K)
    rng = np.random.default_rng(5)
    g = rng.choice([-1, 1], K) * rng.uniform(12, 30, K)
    up = rng.normal(0, 1, K)
    gu = np.concatenate([synth.f64_to_f16_bits(g), synth.f64_to_f16_bits(up)])[None, :]
    y = swiglu_case(eng, rows, gu, N, K)
    assert rel_err(y, oracle.q4_gemv_swiglu(rows, K, gu)) <= TOL
    gu0 = gu.copy()
    gu0[0, K:] = 0
    y0 = swiglu_case(eng, rows, gu0, N, K)
    assert np.all((y0 & 0x7FFF) == 0)


def test_swiglu_deterministic_and_limits(eng):
    N, K = 5120, 17408
    rows = synth.q4_0_matrix(8, synth.weight_id(1), N, K)
    W = packed_on_gpu(eng, rows, N, K)
    gu = f16_dev(synth.activations(8, 1, 2 * K)).reshape(-1)
    a = bits_of(eng.run_swiglu(W, gu, N, K))
    b = bits_of(eng.run_swiglu(W, gu, N, K))
    assert np.array_equal(a, b)
    big = torch.zeros(2 * 65536, dtype=torch.float16, device="cuda")
    y = torch.empty(32, dtype=torch.float16, device="cuda")
    h = eng.h
    st = torch.cuda.current_stream().cuda_stream
    assert q4.q4gemv_run_swiglu(h, W.data_ptr(), big.data_ptr(), y.data_ptr(), 32, 65536, st) == \
        q4.Q4_EUNSUPPORTED
    assert q4.q4gemv_run_swiglu(h, W.data_ptr(), big.data_ptr() + 2, y.data_ptr(), 32, 64, st) == \
        q4.Q4_EALIGN
