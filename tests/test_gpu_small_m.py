"""Q4_0 GEMVs with a few activation vectors (M <= 16) on each small-M kernel,
through the C ABI, against the fp64 oracle.

q4gemv_run sends M = 3..16 (and M <= 2 with K beyond the dp2a kernel's
staging) to the mma.sync kernel; Q4GEMV_SMALL_M=tcs, read when a context is
created, selects the tcgen05 kernel (kind::i8, weights in tensor memory)
instead.  Every engine here must agree with the oracle on
shapes that exercise: one CTA per unit (fewer units than SMs), a row block
whose blocks are split over every CTA (a long K with one row block), ragged
last row blocks and tiles, the 8- and 16-row activation images, extreme codes
and scales, a non-finite input confined to its own vector, and bit-identical
repeats."""
import os

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
KERNELS = ["tcs", "mma"]


@pytest.fixture(scope="module", params=KERNELS)
def eng(request):
    old = os.environ.get("Q4GEMV_SMALL_M")
    os.environ["Q4GEMV_SMALL_M"] = request.param
    try:
        e = q4.Q4Gemv(0)
    finally:
        if old is None:
            os.environ.pop("Q4GEMV_SMALL_M", None)
        else:
            os.environ["Q4GEMV_SMALL_M"] = old
    yield e
    e.close()


def run_case(eng, gguf, x, N, K, M):
    W = packed_on_gpu(eng, gguf, N, K)
    y = eng.run(W, f16_dev(x).reshape(M, K), N, K)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return bits_of(y)


@pytest.mark.parametrize("M", [3, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(1, 32), (33, 64), (257, 160), (1000, 320), (129, 40960),
                                 (40, 6400), (600, 5120)])
def test_small_m_shapes(eng, M, N, K):
    gguf = synth.q4_0_matrix(31 + M, synth.weight_id(3), N, K)
    x = synth.activations(31 + M + K, M, K)
    y = run_case(eng, gguf, x, N, K, M)
    assert rel_err(y, oracle.q4_gemv(gguf, K, x, threads=THREADS)) <= TOL


@pytest.mark.parametrize("M", [4, 16])
@pytest.mark.parametrize("N,K", [(34816, 5120), (5120, 17408)])
def test_small_m_ffn_shapes_sampled(eng, M, N, K):
    gguf = synth.q4_0_matrix(synth.workload_seed(3) + 50 + M, synth.weight_id(0 if K == 5120 else 1), N, K)
    x = synth.activations(synth.workload_seed(3) + 60 + M, M, K)
    y = run_case(eng, gguf, x, N, K, M).reshape(M, N)
    rng = np.random.default_rng(M + K)
    rows = np.unique(np.concatenate([rng.choice(N, 200, replace=False), [0, 127, 128, 255, 256, N - 1]]))
    g = gguf.reshape(N, -1)[rows]
    assert rel_err(np.ascontiguousarray(y[:, rows]), oracle.q4_gemv(g, K, x, threads=THREADS)) <= TOL


def test_extreme_codes_scales_and_nan_confined_to_its_vector(eng):
    N, K, M = 300, 2048, 5
    g = synth.q4_0_matrix(9, synth.weight_id(4), N, K).reshape(N, K // 32, 18)
    g[:, :, 2:] = np.where(np.arange(16) % 2 == 0, 0x0F, 0xF0).astype(np.uint8)   # codes 15 and 0
    g[:, ::3, 0:2] = np.frombuffer(np.float16(1.5).tobytes(), dtype=np.uint8)
    g = g.reshape(N, -1)
    x = synth.activations(9, M, K)
    y = run_case(eng, g, x, N, K, M)
    assert rel_err(y, oracle.q4_gemv(g, K, x)) <= TOL
    xn = x.copy()
    xn[2, 700] = 0x7E00                                   # NaN in vector 2 only
    yn = run_case(eng, g, xn, N, K, M).reshape(M, N).view(np.float16).astype(np.float64)
    assert np.all(np.isnan(yn[2]))
    others = [0, 1, 3, 4]
    assert np.all(np.isfinite(yn[others]))
    assert rel_err(yn[others].astype(np.float16).view(np.uint16), oracle.q4_gemv(g, K, x[others])) <= TOL


@pytest.mark.parametrize("M", [4, 13])
def test_repeat_is_bit_identical(eng, M):
    N, K = 2000, 17408                      # row blocks split over several CTAs
    gguf = synth.q4_0_matrix(12, synth.weight_id(1), N, K)
    x = synth.activations(12, M, K)
    W = packed_on_gpu(eng, gguf, N, K)
    xd = f16_dev(x).reshape(M, K)
    a = bits_of(eng.run(W, xd, N, K))
    b = bits_of(eng.run(W, xd, N, K))
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    assert np.array_equal(a, b)
    assert rel_err(a, oracle.q4_gemv(gguf, K, x, threads=THREADS)) <= TOL


@pytest.mark.parametrize("M", [1, 2])
def test_wide_k_small_m(eng, M):
    """K beyond the dp2a kernel's staging goes to the small-M kernel."""
    N, K = 300, 65536
    gguf = synth.q4_0_matrix(77, synth.weight_id(0), N, K)
    x = synth.activations(77, M, K)
    y = run_case(eng, gguf, x, N, K, M)
    assert rel_err(y, oracle.q4_gemv(gguf, K, x, threads=THREADS)) <= TOL
