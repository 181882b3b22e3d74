"""Parity of the M = 17..256 path (tcgen05 tensor-core GEMM) through the C ABI
against the fp64 oracle: ragged and tiny shapes in full, the pages' prefill
widths (86- and 169-token prompts) on the gate+up and down shapes on sampled
rows, K splits, NaN propagation, determinism and stream capture.

Each weight enters the tensor cores as two binary16 parts whose sum is the
weight exactly, so only fp32 summation and the output rounding remain."""
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


def run_case(eng, gguf, x, N, K):
    M = x.shape[0]
    W = packed_on_gpu(eng, gguf, N, K)
    y = eng.run(W, f16_dev(x).reshape(M, K), N, K)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    return bits_of(y).reshape(M, N)


@pytest.mark.parametrize("N,K,M", [
    (256, 64, 17),       # one CTA, one K step
    (300, 96, 20),       # ragged N, odd block count (half-filled last step)
    (520, 160, 33),      # three CTAs, the last with one tile
    (5, 32, 256),        # N below one tile, widest MMA
    (31, 1056, 100),     # K splits over a single CTA
    (1024, 1024, 86),    # 4 CTAs x 16 splits
    (2048, 5120, 169),
    (96, 40960, 48),     # long K, many splits
])
def test_gemm_shapes_full(eng, N, K, M):
    gguf = synth.q4_0_matrix(900 + N + M, synth.weight_id(0), N, K)
    x = synth.activations(900 + K + M, M, K)
    y = run_case(eng, gguf, x, N, K)
    ref = oracle.q4_gemv(gguf, K, x, threads=THREADS)
    err = rel_err(y, ref)
    assert err <= TOL, err


def sampled_rows(N, n=192, seed=0):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 31, 32, 127, 128, 255, 256, N - 257, N - 256, N - 129, N - 33, N - 1]
    rows = np.unique(np.concatenate([rng.choice(N, n, replace=False), edge]))
    return rows[(rows >= 0) & (rows < N)]


@pytest.mark.parametrize("M", [86, 169])
@pytest.mark.parametrize("N,K", [(34816, 5120), (5120, 17408)])
def test_gemm_prefill_widths_full_shapes_sampled(eng, M, N, K):
    """The gate+up and down shapes at the pages' prompt lengths; the oracle
    computes a sample of rows (all vectors) one by one."""
    tid = 0 if K == 5120 else 1
    gguf = synth.q4_0_matrix(synth.workload_seed(3) + M, synth.weight_id(tid), N, K)
    x = synth.activations(synth.workload_seed(3) + 1000 + M, M, K)
    y = run_case(eng, gguf, x, N, K)
    rows = sampled_rows(N, seed=M)
    ref = oracle.q4_gemv(np.ascontiguousarray(gguf[rows]), K, x, threads=THREADS)
    err = rel_err(np.ascontiguousarray(y[:, rows]), ref)
    assert err <= TOL, err


def test_gemm_error_is_output_rounding_only(eng):
    """With exact weights the error left is fp32 summation plus one binary16
    rounding of y (at most 2^-11 relative): far inside TOL, also at K = 32
    where a single rounded weight would already show."""
    for N, K, M, seed in ((640, 2048, 40, 77), (64, 32, 200, 78)):
        gguf = synth.q4_0_matrix(seed, synth.weight_id(3), N, K)
        x = synth.activations(seed + 1, M, K)
        y = run_case(eng, gguf, x, N, K)
        assert rel_err(y, oracle.q4_gemv(gguf, K, x)) <= 5.2e-4


def test_gemm_nan_activation_poisons_its_vector_only(eng):
    N, K, M = 300, 256, 24
    gguf = synth.q4_0_matrix(12, synth.weight_id(0), N, K)
    x = synth.activations(12, M, K)
    x[5, 77] = 0x7E00
    y = run_case(eng, gguf, x, N, K).view(np.float16).astype(np.float64)
    assert np.all(np.isnan(y[5]))
    keep = np.arange(M) != 5
    assert np.all(np.isfinite(y[keep]))
    ref = oracle.q4_gemv(gguf, K, x[keep])
    assert rel_err(y[keep].astype(np.float16).view(np.uint16), ref) <= TOL


def test_gemm_deterministic_bits(eng):
    N, K, M = 5120, 17408, 64
    gguf = synth.q4_0_matrix(13, synth.weight_id(1), N, K)
    x = f16_dev(synth.activations(13, M, K))
    W = packed_on_gpu(eng, gguf, N, K)
    a = bits_of(eng.run(W, x, N, K))
    b = bits_of(eng.run(W, x, N, K))
    assert np.array_equal(a, b)


def test_gemm_user_stream_capture(eng):
    N, K, M = 1024, 2048, 32
    gguf = synth.q4_0_matrix(14, synth.weight_id(0), N, K)
    x = synth.activations(14, M, K)
    W = packed_on_gpu(eng, gguf, N, K)
    xd = f16_dev(x).reshape(M, K)
    y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    eng.run(W, xd, N, K, out=y)          # first call sizes the workspace
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        eng.run(W, xd, N, K, out=y)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert rel_err(bits_of(y), oracle.q4_gemv(gguf, K, x, threads=THREADS)) <= TOL
