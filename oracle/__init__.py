"""ORACLE -- test infrastructure only.

Plain fp64 CPU restatement of the Q4_0 dequantise-and-multiply GEMV, the
repack layout, the renormalised layer chain and the SiLU-gated input of the
down GEMV (see ``q4_oracle.c`` for the citations and readings).  Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference leg may import this package; the CUDA product path
never does and shares no code with it.

Every function here is pinned in ``tests/test_oracle_pins.py`` (SiLU gating:
``tests/test_oracle_swiglu_pins.py``).  The layer
chain (``stack_step``) is pinned by signed-permutation stacks whose result has
a closed form.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile q4_oracle.c into liboracle.so (gcc -O2, no fused FP ops)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _configure(lib):
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_f64.restype = ctypes.c_double
    lib.oracle_f64_to_f16.argtypes = [ctypes.c_double]
    lib.oracle_f64_to_f16.restype = ctypes.c_uint16
    lib.oracle_q4_gemv.argtypes = [vp, i64, i64, vp, i64, vp]
    lib.oracle_q4_gemv.restype = None
    lib.oracle_repack.argtypes = [vp, i64, i64, vp]
    lib.oracle_repack.restype = None
    lib.oracle_renorm.argtypes = [vp, i64, vp]
    lib.oracle_renorm.restype = None
    lib.oracle_q8_gemv.argtypes = [vp, i64, i64, vp, i64, vp]
    lib.oracle_q8_gemv.restype = None
    lib.oracle_repack_q8.argtypes = [vp, i64, i64, vp]
    lib.oracle_repack_q8.restype = None
    lib.oracle_unit_rms_scale.argtypes = [vp, i64]
    lib.oracle_unit_rms_scale.restype = ctypes.c_double
    lib.oracle_round_f16.argtypes = [vp, i64, vp]
    lib.oracle_round_f16.restype = None
    lib.oracle_swiglu.argtypes = [vp, i64, i64, vp]
    lib.oracle_swiglu.restype = None
    lib.oracle_q4_gemv_f64.argtypes = [vp, i64, i64, vp, i64, vp]
    lib.oracle_q4_gemv_f64.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _swap_library(path):
    """Point this module at another build of q4_oracle.c (used by the
    mutation test, which plants mistakes in a copy of the source); returns
    the previous library handle so it can be restored."""
    global _lib
    with _lock:
        prev = _lib
        _lib = _configure(ctypes.CDLL(path)) if path is not None else None
    return prev


def _restore_library(prev):
    global _lib
    with _lock:
        _lib = prev


def f16_to_f64(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.oracle_f16_to_f64(int(v)) for v in b.ravel()],
                    dtype=np.float64).reshape(b.shape)


def f64_to_f16(v) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_round_f16(a.ctypes.data, a.size, out.ctypes.data)
    return out


def q4_gemv(rows: np.ndarray, K: int, x: np.ndarray, threads: int = 1) -> np.ndarray:
    """y[M][nrows] (fp64) for GGUF rows (nrows, K/32*18) uint8 and x[M][K]
    f16 bit patterns.  ``threads`` > 1 splits the rows across threads."""
    return _gemv(_load().oracle_q4_gemv, 18, rows, K, x, threads)


def q8_gemv(rows: np.ndarray, K: int, x: np.ndarray, threads: int = 1) -> np.ndarray:
    """As q4_gemv, for GGUF Q8_0 rows (nrows, K/32*34) uint8."""
    return _gemv(_load().oracle_q8_gemv, 34, rows, K, x, threads)


def _gemv(fn, block_bytes: int, rows: np.ndarray, K: int, x: np.ndarray, threads: int) -> np.ndarray:
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    M = x.shape[0]
    assert x.shape[1] == K and K % 32 == 0
    rb = (K // 32) * block_bytes
    nrows = rows.size // rb
    assert rows.size == nrows * rb
    y = np.empty((M, nrows), dtype=np.float64)
    if threads <= 1 or nrows < 2 * threads:
        fn(rows.ctypes.data, nrows, K, x.ctypes.data, M, y.ctypes.data)
        return y
    # partition rows; each worker writes its own [M][chunk] block
    bounds = np.linspace(0, nrows, threads + 1).astype(np.int64)
    parts = [np.empty((M, int(bounds[i + 1] - bounds[i])), dtype=np.float64)
             for i in range(threads)]

    def work(i):
        r0, r1 = int(bounds[i]), int(bounds[i + 1])
        if r1 > r0:
            fn(rows.ctypes.data + r0 * rb, r1 - r0, K, x.ctypes.data, M, parts[i].ctypes.data)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(threads)))
    return np.concatenate(parts, axis=1)


def swiglu(gate_up: np.ndarray) -> np.ndarray:
    """u[M][K] = SiLU(gate) * up (fp64) for f16 bit patterns [M][2K] laid out
    as [gate | up] (see ``q4_oracle.c`` for the reading)."""
    v = np.ascontiguousarray(np.atleast_2d(gate_up), dtype=np.uint16)
    M, K2 = v.shape
    assert K2 % 2 == 0
    u = np.empty((M, K2 // 2), dtype=np.float64)
    _load().oracle_swiglu(v.ctypes.data, K2 // 2, M, u.ctypes.data)
    return u


def q4_gemv_f64(rows: np.ndarray, K: int, x: np.ndarray, threads: int = 1) -> np.ndarray:
    """As q4_gemv with an fp64 input x[M][K]."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    M = x.shape[0]
    assert x.shape[1] == K and K % 32 == 0
    rb = (K // 32) * 18
    nrows = rows.size // rb
    assert rows.size == nrows * rb
    fn = _load().oracle_q4_gemv_f64
    if threads <= 1 or nrows < 2 * threads:
        y = np.empty((M, nrows), dtype=np.float64)
        fn(rows.ctypes.data, nrows, K, x.ctypes.data, M, y.ctypes.data)
        return y
    bounds = np.linspace(0, nrows, threads + 1).astype(np.int64)
    parts = [np.empty((M, int(bounds[i + 1] - bounds[i])), dtype=np.float64) for i in range(threads)]

    def work(i):
        r0, r1 = int(bounds[i]), int(bounds[i + 1])
        if r1 > r0:
            fn(rows.ctypes.data + r0 * rb, r1 - r0, K, x.ctypes.data, M, parts[i].ctypes.data)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(threads)))
    return np.concatenate(parts, axis=1)


def q4_gemv_swiglu(rows: np.ndarray, K: int, gate_up: np.ndarray, threads: int = 1) -> np.ndarray:
    """y = W (SiLU(gate) * up): the down GEMV fed by the gate+up output."""
    return q4_gemv_f64(rows, K, swiglu(gate_up), threads)


def packed_bytes(N: int, K: int) -> int:
    Np = (N + 31) // 32 * 32
    return Np * (K // 32) * 18


def repack(gguf: np.ndarray, N: int, K: int) -> np.ndarray:
    out = np.empty(packed_bytes(N, K), dtype=np.uint8)
    g = np.ascontiguousarray(gguf, dtype=np.uint8)
    assert g.size == N * (K // 32) * 18
    _load().oracle_repack(g.ctypes.data, N, K, out.ctypes.data)
    return out


def packed_bytes_q8(N: int, K: int) -> int:
    Np = (N + 31) // 32 * 32
    return Np * (K // 32) * 34


def repack_q8(gguf: np.ndarray, N: int, K: int) -> np.ndarray:
    out = np.empty(packed_bytes_q8(N, K), dtype=np.uint8)
    g = np.ascontiguousarray(gguf, dtype=np.uint8)
    assert g.size == N * (K // 32) * 34
    _load().oracle_repack_q8(g.ctypes.data, N, K, out.ctypes.data)
    return out


def renorm(v: np.ndarray) -> np.ndarray:
    """f16(v * unit_rms_scale(v)): the step's final output vector."""
    v = np.ascontiguousarray(v, dtype=np.uint16)
    out = np.empty_like(v)
    _load().oracle_renorm(v.ctypes.data, v.size, out.ctypes.data)
    return out


def unit_rms_scale(v: np.ndarray) -> float:
    """1 / sqrt(mean(v^2)) of an f16 vector in fp64 (0 for an all-zero one)."""
    v = np.ascontiguousarray(v, dtype=np.uint16)
    return float(_load().oracle_unit_rms_scale(v.ctypes.data, v.size))


def stack_step(get_rows, x_in: np.ndarray, n_layers: int, hidden: int,
               qkv_n: int, ffn: int, threads: int = 1, record=None, gated: bool = False):
    """The renormalised 64-layer-style chain of GEMVs (one decode step, M=1).

    Layer l, with matrices QKV (qkv_n x hidden), O (hidden x hidden),
    gate+up (2*ffn x hidden), down (hidden x ffn), each GEMV output rounded
    to f16 (the boundary's vector type) and each next input taken as that
    f16 vector (its first K entries) scaled to unit RMS by a real scalar:
        a = f16(QKV x);           b = f16(O (s(a') a'))       a' = a[0:hidden]
        u = f16(gate_up (s(b) b)); x' = f16(down (s(u') u'))  u' = u[0:ffn]
    with s(v) = 1/sqrt(mean(v^2)) (0 for v = 0); by linearity each output
    is f16(s * (W v)), computed here in fp64.  The step returns the next
    layer's input as an f16 vector, f16(s(x') x').  ``get_rows(l, t)``
    returns the GGUF bytes of matrix t (0 QKV, 1 O, 2 gate+up, 3 down) of
    layer l.  ``record(i, x_f16, s, y_f64)`` is called for each GEMV
    i = 4l + t when given (x_f16: the unscaled input, s its scale, y_f64 the
    output before rounding).

    ``gated``: the FFN with its activation -- the down GEMV's input is
    u = SiLU(gate) * up of the whole f16 gate+up output (``swiglu``: gate
    half first, fp64, never rounded), scaled to unit RMS like every input of
    the chain: x' = f16(s(u) (down u)), s(u) = 1/sqrt(mean(u^2)) in fp64 (0
    for u = 0).  ``record`` then gets the 2*ffn-entry gate+up vector as the
    down GEMV's input.
    """
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    x = np.ascontiguousarray(x_in, dtype=np.uint16)
    s = 1.0
    for l in range(n_layers):
        for t, (N, K) in enumerate(dims):
            if gated and t == 3:
                assert x.size == 2 * K
                u = swiglu(x.reshape(1, 2 * K))[0]
                ms = float(np.mean(u * u))
                s = 1.0 / np.sqrt(ms) if ms > 0 else 0.0
                with np.errstate(invalid="ignore"):
                    y = s * q4_gemv_f64(get_rows(l, t), K, u.reshape(1, K), threads=threads)[0]
            else:
                assert x.size == K
                with np.errstate(invalid="ignore"):      # 0 * inf of a non-finite row is NaN
                    y = s * q4_gemv(get_rows(l, t), K, x.reshape(1, K), threads=threads)[0]
            if record is not None:
                record(4 * l + t, x, s, y)
            yh = f64_to_f16(y)
            keep = {0: hidden, 1: hidden, 2: 2 * ffn if gated else ffn, 3: hidden}[t]
            x = np.ascontiguousarray(yh[:keep])
            s = unit_rms_scale(x)
    return renorm(x)
