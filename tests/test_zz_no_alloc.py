"""q4gemv_run_noalloc on the GPU, through the C ABI.

Some callers cannot allocate device memory (for example code that runs while
a stream is captured in global mode, or a plug-in whose host application
owns all device memory); for them the library offers a GEMV entry point whose
scratch lives in a fixed device array instead of a cudaMalloc'd workspace.
This file checks that two calls in a row each match the fp64 oracle and
q4gemv_run within the GEMV tolerance, and that sizes beyond the array's
limits are refused.  It is named so that pytest collects it last."""
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


@pytest.mark.parametrize("M,N,K", [(1, 5120, 5120), (1, 34816, 5120), (1, 5120, 17408),
                                   (2, 4096, 5120), (1, 33, 64)])
def test_noalloc_matches_run_twice(M, N, K):
    eng = q4.Q4Gemv(0)
    gguf = synth.q4_0_matrix(606 + N, synth.weight_id(0), N, K)
    W = packed_on_gpu(eng, gguf, N, K)
    xb = synth.activations(606 + K, M, K)
    x = f16_dev(xb).reshape(M, K)
    exact = oracle.q4_gemv(gguf, K, xb, threads=8)
    ref = eng.run(W, x, N, K)
    st = q4._stream(None)
    for _ in range(2):
        y = torch.full((M, N), 3.0, dtype=torch.float16, device="cuda")
        rc = q4.q4gemv_run_noalloc(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, st)
        assert rc == q4.Q4_OK
        torch.cuda.synchronize()
        err = rel_err(bits_of(y), exact)
        assert err <= TOL, err
        err = rel_err(bits_of(y), bits_of(ref).view(np.float16).astype(np.float64))
        assert err <= TOL, err
    assert eng.sync_status() == q4.Q4_OK
    eng.close()


def test_noalloc_rejects_sizes_beyond_its_limits():
    st = q4._stream(None)
    buf = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    assert q4.q4gemv_run_noalloc(p, p, p, 3, 32, 32, st) == q4.Q4_EUNSUPPORTED
    assert q4.q4gemv_run_noalloc(p, p, p, 1, (1 << 22) + 32, 32, st) == q4.Q4_ESHAPE
    assert q4.q4gemv_run_noalloc(p, p, p, 1, 32, 40960, st) == q4.Q4_ESHAPE
    assert q4.q4gemv_run_noalloc(p, p, p, 2, 32, 20480, st) == q4.Q4_ESHAPE
    assert q4.q4gemv_run_noalloc(p, p, p, 1, 32, 48, st) == q4.Q4_ESHAPE
    assert q4.q4gemv_run_noalloc(p + 8, p, p, 1, 32, 32, st) == q4.Q4_EALIGN


@pytest.mark.parametrize("M,K_ok", [(1, 24896), (2, 18432)])
def test_noalloc_largest_k(M, K_ok):
    """The largest K each M accepts runs; one block more is refused."""
    N = 64
    st = q4._stream(None)
    gguf = synth.q4_0_matrix(17, synth.weight_id(0), N, K_ok)
    eng = q4.Q4Gemv(0)
    W = packed_on_gpu(eng, gguf, N, K_ok)
    xb = synth.activations(18, M, K_ok)
    x = f16_dev(xb).reshape(M, K_ok)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert q4.q4gemv_run_noalloc(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K_ok, st) == q4.Q4_OK
    torch.cuda.synchronize()
    assert rel_err(bits_of(y), oracle.q4_gemv(gguf, K_ok, xb, threads=8)) <= TOL
    big = torch.empty(4 << 20, dtype=torch.uint8, device="cuda")
    p = big.data_ptr()
    assert q4.q4gemv_run_noalloc(p, p, p, M, N, K_ok + 32, st) == q4.Q4_ESHAPE
    eng.close()
