"""C-ABI checks that need no GPU: the library loads, exports every entry
point declared in include/q4gemv.h, and rejects bad arguments on the host."""
import ctypes
import os
import re

import pytest

import q4_quantized_decode_b200 as q4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q4gemv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(q4gemv_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["q4gemv_create", "q4gemv_destroy", "q4gemv_repack", "q4gemv_run",
              "q4gemv_run_stack", "q4gemv_packed_bytes", "q4gemv_strerror"]:
        assert n in names


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(q4.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_version_and_strerror():
    assert q4.q4gemv_version() >= 1
    for st in [0, -1, -2, -3, -4, -5, -6, -7, -8, -9]:
        assert q4.q4gemv_strerror(st) != "unknown status"
    assert q4.q4gemv_strerror(12345) == "unknown status"


@pytest.mark.parametrize("N,K", [(1024, 1024), (5120, 5120), (34816, 5120), (5120, 17408),
                                 (7168, 5120), (1, 32), (33, 64)])
def test_sizes(N, K):
    Np = (N + 31) // 32 * 32
    assert q4.q4gemv_gguf_bytes(N, K) == N * (K // 32) * 18
    assert q4.q4gemv_packed_bytes(N, K) == Np * (K // 32) * 18


@pytest.mark.parametrize("N,K", [(0, 32), (32, 0), (32, 48), (-1, 32), (32, -32),
                                 ((1 << 22) + 1, 32), (32, (1 << 20) + 32)])
def test_bad_shapes_have_zero_size(N, K):
    assert q4.q4gemv_gguf_bytes(N, K) == 0
    assert q4.q4gemv_packed_bytes(N, K) == 0


A = 1 << 20  # a 16-byte aligned fake address (never dereferenced)


def test_validate_paths():
    v = q4.q4gemv_validate
    assert v(1, 5120, 5120, A, A, A) == q4.Q4_OK
    assert v(2, 5120, 17408, A, A, A) == q4.Q4_OK
    assert v(0, 32, 32, A, A, A) == q4.Q4_EUNSUPPORTED
    assert v(17, 32, 32, A, A, A) == q4.Q4_OK          # tensor-core GEMM path
    assert v(256, 32, 32, A, A, A) == q4.Q4_OK
    assert v(257, 32, 32, A, A, A) == q4.Q4_EUNSUPPORTED
    assert v(1, 32, 48, A, A, A) == q4.Q4_ESHAPE
    assert v(1, 0, 32, A, A, A) == q4.Q4_ESHAPE
    assert v(1, 32, 32, None, A, A) == q4.Q4_EINVAL
    assert v(1, 32, 32, A, None, A) == q4.Q4_EINVAL
    assert v(1, 32, 32, A, A, None) == q4.Q4_EINVAL
    assert v(1, 32, 32, A + 8, A, A) == q4.Q4_EALIGN
    assert v(1, 32, 32, A, A + 2, A) == q4.Q4_EALIGN
    assert v(1, 32, 32, A, A, A + 4) == q4.Q4_EALIGN


def test_validate_accepts_wide_tensor_core_shapes():
    """Matrices wider than one CTA's activation staging run as column panels,
    so validation accepts them within the general limits."""
    v = q4.q4gemv_validate
    assert v(1, 32, 1 << 17, A, A, A) == q4.Q4_OK
    assert v(4, 4096, 1 << 17, A, A, A) == q4.Q4_OK
    assert v(1, 1 << 20, 1 << 17, A, A, A) == q4.Q4_OK
    assert v(16, 1 << 16, 1 << 16, A, A, A) == q4.Q4_OK
    assert v(16, 1 << 22, 1 << 20, A, A, A) == q4.Q4_ESHAPE   # ceil(N/32) * K/32 >= 2^31


def test_null_handle_is_rejected():
    assert q4.q4gemv_run(None, A, A, A, 1, 32, 32, None) == q4.Q4_EINVAL
    assert q4.q4gemv_repack(None, A, A, 32, 32, None) == q4.Q4_EINVAL
    assert q4.q4gemv_sync_status(None, None) == q4.Q4_EINVAL
    assert q4.q4gemv_set_fault(None, "alloc") == q4.Q4_EINVAL
    assert q4.q4gemv_destroy(None) == q4.Q4_OK
    assert q4.q4gemv_last_error(None) == ""
